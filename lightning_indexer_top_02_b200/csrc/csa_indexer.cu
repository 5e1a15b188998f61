// csa_indexer.cu -- host side of the C ABI declared in include/csa_indexer.h:
// argument validation, work planning (query blocks, key splits, pipeline
// depth, candidate capacity, launch chunks), TMA descriptors, workspace layout
// and the launches: per chunk of query blocks, the fused scoring/filter kernel
// and then the exact top-k selection over its candidate lists.
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "csa_indexer.h"
#include "indexer_kernel.cuh"
#include "select_kernel.cuh"
#include "sparse_attn_kernel.cuh"
#include "union_kernel.cuh"

namespace {

using csa::Params;

constexpr int kVersion = 100; // 0.1.0
constexpr int kSmemLimit = 232448; // 227 KB of dynamic shared memory per CTA on sm_100
constexpr unsigned long long kDefaultWaitLimit = 4000000000ull;

unsigned long long g_wait_limit = kDefaultWaitLimit;

// NVTX range around a host-side region (a profiler's timeline shows each
// call and each launch chunk by name; without a profiler attached the calls
// are no-ops).
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

// Measurement hook: events recorded around this thread's launches.
thread_local cudaEvent_t *t_events = nullptr;
thread_local int t_n_events = 0;

// Records event j of the current call, if the caller asked for it.
bool mark(int j, cudaStream_t stream)
{
    if (j >= t_n_events)
        return true;
    return cudaEventRecord(t_events[j], stream) == cudaSuccess;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

int pow2_ceil(long long x)
{
    int p = 1;
    while (p < x && p < (1 << 30))
        p <<= 1;
    return p;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Workspace the default entry points may use for one launch chunk; larger
// problems run as several chunks of query blocks.
constexpr size_t kDefaultWorkspaceCap = size_t(16) << 30;

struct Plan {
    Params p;          // qb_lo, nqb and n_items describe the first chunk
    int grid;
    int nqb_total;     // query blocks per batch
    int qb_chunk;      // query blocks per batch in one launch chunk
    int chunks;
    int fast_fc, fast_fq; // epilogue fast path (0 = generic)
    size_t ws_lists, ws_counts, ws_scores, ws_total;
};

csa_status_t validate(const csa_args_t *a)
{
    if (!a)
        return CSA_ERR_INVALID_ARG;
    if (a->B < 0 || a->S < 0 || a->T < 0 || a->H_I <= 0 || a->d <= 0 || a->m <= 0 ||
        a->topk <= 0)
        return CSA_ERR_INVALID_ARG;
    if ((a->causal != 0 && a->causal != 1) || (a->mode != CSA_MODE_TOPK && a->mode != CSA_MODE_GATE) ||
        (a->key_dtype != CSA_KEY_BF16 && a->key_dtype != CSA_KEY_E4M3))
        return CSA_ERR_INVALID_ARG;
    if (a->query_pieces < 0 || a->query_pieces > 2 ||
        (a->key_dtype == CSA_KEY_BF16 && a->query_pieces != 0))
        return CSA_ERR_INVALID_ARG;
    if (static_cast<long long>(a->B) * a->S == 0)
        return CSA_OK;
    if (!a->q || !a->w || !a->out_idx || !a->out_score)
        return CSA_ERR_INVALID_ARG;
    if (a->T > 0 && !a->k)
        return CSA_ERR_INVALID_ARG;
    if (a->key_dtype == CSA_KEY_E4M3 && a->T > 0 && !a->k_scale)
        return CSA_ERR_INVALID_ARG;
    if (!aligned(a->q, 16) || (a->k && !aligned(a->k, 16)) || !aligned(a->w, 4) ||
        !aligned(a->out_idx, 4) || !aligned(a->out_score, 4) ||
        (a->k_scale && !aligned(a->k_scale, 4)))
        return CSA_ERR_INVALID_ARG;
    if (a->q_offset != CSA_Q_OFFSET_DEFAULT &&
        (a->q_offset < -(1ll << 62) || a->q_offset > (1ll << 62)))
        return CSA_ERR_INVALID_ARG;
    if (!is_pow2(a->H_I) || a->H_I > 256)
        return CSA_ERR_UNSUPPORTED;
    if (a->d != 32 && a->d != 64 && a->d != 128)
        return CSA_ERR_UNSUPPORTED;
    if (a->topk > csa::kMaxTopk)
        return CSA_ERR_UNSUPPORTED;
    const long long rows_q = static_cast<long long>(a->B) * a->S * a->H_I;
    const long long rows_k = static_cast<long long>(a->B) * a->T;
    if (rows_q >= (1ll << 31) || rows_k >= (1ll << 31))
        return CSA_ERR_UNSUPPORTED;
    return CSA_OK;
}

int device_sms()
{
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 0;
    return sms;
}

// Number of key tiles the heaviest query block of a batch touches.
int max_tiles(const csa_args_t *a, long long q_offset)
{
    long long nvis = a->T;
    if (a->causal) {
        const long long t = static_cast<long long>(a->S) - 1 + q_offset;
        nvis = (t + 1) / a->m;
        if (nvis > a->T)
            nvis = a->T;
        if (nvis < 0)
            nvis = 0;
    }
    return static_cast<int>((nvis + csa::kTileKeys - 1) / csa::kTileKeys);
}

csa_status_t make_plan(const csa_args_t *a, int sms, size_t ws_cap, Plan *out)
{
    Params p;
    std::memset(&p, 0, sizeof p);
    p.B = a->B;
    p.S = a->S;
    p.T = a->T;
    p.H = a->H_I;
    p.d = a->d;
    p.m = a->m;
    p.topk = a->topk;
    p.causal = a->causal;
    p.mode = a->mode;
    p.key_fp8 = a->key_dtype == CSA_KEY_E4M3;
    p.q_pieces = p.key_fp8 ? (a->query_pieces == 1 ? 1 : 2) : 0;
    p.q_offset = a->q_offset != CSA_Q_OFFSET_DEFAULT ? a->q_offset
                                  : (static_cast<long long>(a->T) * a->m > a->S
                                         ? static_cast<long long>(a->T) * a->m - a->S
                                         : 0);
    p.row_bytes = a->d * 2 < 128 ? a->d * 2 : 128;
    p.n_chunks = a->d * 2 / p.row_bytes;

    // Query block: as many queries as fill 256 MMA columns, no more than S
    // needs, and at least 32 columns (one TMEM load of the epilogue).
    int qps = 256 / p.H;
    if (qps > pow2_ceil(p.S))
        qps = pow2_ceil(p.S);
    if (qps * p.H < 32)
        qps = 32 / p.H;
    p.qps = qps;
    p.N = qps * p.H;
    // Two epilogue warpgroups split the queries when each half still spans
    // whole 32-column TMEM loads.
    p.n_wg = (qps >= 2 && p.N >= 64) ? 2 : 1;
    p.qpw = qps / p.n_wg;
    // One query per item: both warpgroups read every column and take
    // alternate key tiles instead of splitting the queries.
    p.tile_split = qps == 1 ? 1 : 0;
    if (p.tile_split)
        p.n_wg = 2;
    // Small N: several key tiles share one accumulator slot, side by side.
    p.tpg = csa::kSlotCols / p.N < csa::kMaxTpg ? csa::kSlotCols / p.N : csa::kMaxTpg;

    // Candidate list per (query, split): the top k plus room for the
    // selector's histogram bucket around the k-th score.
    int extra = p.topk / 4;
    if (extra < 256)
        extra = 256;
    p.cap = (p.topk + extra + 127) / 128 * 128;

    // Shared memory: the bf16 query block (where the TMA lands it), with E4M3
    // keys its two E4M3 pieces (hi8 and lo8 blocks of N rows x d bytes), the
    // ring of key tiles (bf16, or E4M3 as stored) with every stage that fits,
    // then weights, query scales, selector scratch and barriers.
    const int ktile = csa::kTileKeys * p.d * (p.key_fp8 ? 1 : 2);
    int off = 0;
    p.off_q = off;
    off += p.N * p.d * 2;
    if (p.key_fp8) {
        p.off_e = off;
        off += p.q_pieces * p.N * p.d;
    }
    p.off_k = off;
    const int w_bytes = 4 * p.qps * p.H * 4;           // w: per item parity (and group)
    const int sig_bytes = p.key_fp8 ? 2 * p.N * 4 : 0;  // query scales: per item parity
    int tail = (w_bytes + sig_bytes + 15) / 16 * 16;
    tail += (static_cast<int>(sizeof(csa::SelectorScratch)) + 15) / 16 * 16;
    tail += static_cast<int>(sizeof(csa::Barriers)) + 16;
    const int room = kSmemLimit - 1024 - off - tail;
    int stages = room / ktile;
    if (stages > csa::kMaxStages)
        stages = csa::kMaxStages;
    if (stages < 2)
        return CSA_ERR_UNSUPPORTED;
    p.stages = stages;
    off += stages * ktile;
    p.off_w = off;
    off += w_bytes;
    p.off_sig = off;
    off += sig_bytes;
    off = (off + 15) / 16 * 16;
    p.off_sel = off;
    off += (static_cast<int>(sizeof(csa::SelectorScratch)) + 15) / 16 * 16;
    p.off_bar = off;
    off += static_cast<int>(sizeof(csa::Barriers));
    p.smem_bytes = off + 1024;
    // More than half of the SM's shared memory: one CTA per SM, so the CTA's
    // 512-column TMEM allocation never waits on a neighbour.
    if (p.smem_bytes < kSmemLimit / 2 + 1024)
        p.smem_bytes = kSmemLimit / 2 + 1024;
    const int nqb_total = (p.S + p.qps - 1) / p.qps;

    // Key-range splits: only when there are too few query blocks to fill the
    // GPU; pick the count with the best last-wave occupancy.
    const long long items_base = static_cast<long long>(p.B) * nqb_total;
    int nsplit = 1;
    if (a->num_splits > 0) {
        nsplit = a->num_splits;
    } else if (items_base < 4ll * sms) {
        const int tiles = max_tiles(a, p.q_offset);
        int max_split = 16;
        if (max_split > tiles)
            max_split = tiles;
        double best = -1.0;
        for (int s = 1; s <= max_split; ++s) {
            const long long items = items_base * s;
            const long long waves = (items + sms - 1) / sms;
            const double eff = static_cast<double>(items) / static_cast<double>(waves * sms);
            const double score = eff - 0.01 * (s - 1);
            if (score > best + 1e-9) {
                best = score;
                nsplit = s;
            }
        }
    }
    const int tiles_max = max_tiles(a, p.q_offset);
    // Longer key ranges split into items of at most max_item keys, so that an
    // item's score buffer (qps x keys fp32, two per CTA) is re-read by the
    // selector from L2 rather than HBM.  Each split adds a candidate list per
    // query for the select kernel, which costs little when there are few query
    // rows (decode): then items stop at 16,384 keys, else at kMaxItemKeys.
    const long long rows_total = static_cast<long long>(p.B) * p.S;
    int max_item = rows_total <= 16384 ? 16384 : csa::kMaxItemKeys;
    if ((tiles_max * csa::kTileKeys + max_item - 1) / max_item > csa::kSelMaxSplits)
        max_item = csa::kMaxItemKeys;
    const int min_split = (tiles_max * csa::kTileKeys + max_item - 1) / max_item;
    if (nsplit < min_split)
        nsplit = min_split;
    if (nsplit < 1 || nsplit > csa::kSelMaxSplits)
        return CSA_ERR_UNSUPPORTED;
    p.nsplit = nsplit;
    // keys of the longest item: its split's share of the heaviest query block's tiles
    p.nmax = (tiles_max + nsplit - 1) / nsplit * csa::kTileKeys;
    if (p.nmax < csa::kTileKeys)
        p.nmax = csa::kTileKeys;

    // Score buffers: per CTA two halves of qps x nmax fp32 (grid-sized, not
    // S-sized).  A budget that cannot hold a full grid's buffers next to one
    // query block's lists runs fewer CTAs.
    int grid = sms;
    const size_t scores_per_cta = static_cast<size_t>(2) * p.qps * p.nmax * 4;
    // Candidate lists: one per (query, split), cap keys each, plus its length.
    // A launch chunk covers qb_chunk query blocks of every batch.
    const size_t rows_per_qb = static_cast<size_t>(p.B) * p.qps;
    const size_t lists_per_qb = rows_per_qb * nsplit * p.cap * 8;
    const size_t counts_per_qb = rows_per_qb * nsplit * 4;
    const size_t per_qb = lists_per_qb + counts_per_qb;
    if (static_cast<size_t>(grid) * scores_per_cta + per_qb + 1024 > ws_cap) {
        if (ws_cap < per_qb + scores_per_cta + 1024)
            return CSA_ERR_WORKSPACE;
        const size_t fit = (ws_cap - per_qb - 1024) / scores_per_cta;
        grid = static_cast<int>(fit < static_cast<size_t>(grid) ? fit : grid);
    }
    const size_t ws_scores = align256(static_cast<size_t>(grid) * scores_per_cta);
    long long qb_chunk = nqb_total;
    if (static_cast<size_t>(qb_chunk) * per_qb + ws_scores + 1024 > ws_cap)
        qb_chunk = static_cast<long long>((ws_cap - ws_scores - 1024) / per_qb);
    if (qb_chunk < 1)
        return CSA_ERR_WORKSPACE;
    const long long items = static_cast<long long>(p.B) * qb_chunk * nsplit;
    if (items >= (1ll << 31) || static_cast<long long>(p.B) * qb_chunk * p.qps >= (1ll << 31))
        return CSA_ERR_UNSUPPORTED;
    p.qb_lo = 0;
    p.nqb = static_cast<int>(qb_chunk);
    p.n_items = static_cast<int>(items);

    Plan plan;
    plan.nqb_total = nqb_total;
    plan.qb_chunk = static_cast<int>(qb_chunk);
    plan.chunks = static_cast<int>((nqb_total + qb_chunk - 1) / qb_chunk);
    plan.grid = p.n_items < grid ? p.n_items : grid;
    if (plan.grid < 1)
        plan.grid = 1;
    plan.ws_lists = align256(static_cast<size_t>(qb_chunk) * lists_per_qb);
    plan.ws_counts = align256(static_cast<size_t>(qb_chunk) * counts_per_qb);
    plan.ws_scores = ws_scores;
    plan.ws_total = plan.ws_lists + plan.ws_counts + plan.ws_scores;
    // Epilogue fast path: whole 32-column queries, 64 or 128 columns per group.
    const int cols = p.qpw * p.H;
    plan.fast_fc = (p.H >= 32 && (cols == 64 || cols == 128)) ? cols : 0;
    plan.fast_fq = plan.fast_fc ? p.qpw : 0;
    plan.p = p;
    *out = plan;
    return CSA_OK;
}

bool make_tmap(CUtensorMap *tm, CUtensorMapDataType dt, const void *base, long long rows, int cols,
               int box_cols, int box_rows, CUtensorMapSwizzle swz, int elem_bytes = 2,
               long long row_stride = 0)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc)
        return false;
    const cuuint64_t gdim[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    const cuuint64_t gstride[1] = {static_cast<cuuint64_t>(row_stride > 0 ? row_stride : cols) *
                                   elem_bytes};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estride[2] = {1, 1};
    return enc(tm, dt, 2, const_cast<void *>(base), gdim, gstride, box, estride,
               CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

__global__ void pad_outputs_kernel(int32_t *idx, float *score, long long n)
{
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        idx[i] = -1;
        score[i] = -__int_as_float(0x7f800000);
    }
}

using KernelFn = void (*)(const CUtensorMap, const CUtensorMap, const Params);

KernelFn pick_kernel(const Plan &plan)
{
    switch (plan.fast_fc * 8 + plan.fast_fq) {
    case 64 * 8 + 1: return csa::indexer_topk_kernel<64, 1, true>;
    case 64 * 8 + 2: return csa::indexer_topk_kernel<64, 2, true>;
    case 128 * 8 + 1: return csa::indexer_topk_kernel<128, 1, true>;
    case 128 * 8 + 2: return csa::indexer_topk_kernel<128, 2, true>;
    case 128 * 8 + 4: return csa::indexer_topk_kernel<128, 4, true>;
    default: break;
    }
    return plan.p.H >= 32 ? csa::indexer_topk_kernel<0, 0, true>
                          : csa::indexer_topk_kernel<0, 0, false>;
}

csa_status_t launch(const csa_args_t *a, const Plan &plan, void *ws, cudaStream_t stream)
{
    Params p = plan.p;
    p.q = static_cast<const uint16_t *>(a->q);
    p.w = a->w;
    p.k_scale = a->k_scale;
    p.lists = reinterpret_cast<uint64_t *>(ws);
    p.counts = reinterpret_cast<int *>(static_cast<uint8_t *>(ws) + plan.ws_lists);
    p.scores = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + plan.ws_lists + plan.ws_counts);
    p.wait_limit = static_cast<long long>(g_wait_limit);

    CUtensorMap tmQ, tmK;
    const CUtensorMapSwizzle swz =
        p.row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    const CUtensorMapDataType qdt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    if (!make_tmap(&tmQ, qdt, a->q, static_cast<long long>(p.B) * p.S * p.H, p.d, p.row_bytes / 2,
                   p.N, swz))
        return CSA_ERR_CUDA;
    if (p.key_fp8) {
        // E4M3 rows of d bytes, swizzled at that width: the MMA's A operand as is
        const CUtensorMapSwizzle swz8 = p.d == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                        : p.d == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                    : CU_TENSOR_MAP_SWIZZLE_32B;
        if (!make_tmap(&tmK, CU_TENSOR_MAP_DATA_TYPE_UINT8, a->k, static_cast<long long>(p.B) * p.T,
                       p.d, p.d, csa::kTileKeys, swz8, 1))
            return CSA_ERR_CUDA;
    } else if (!make_tmap(&tmK, qdt, a->k, static_cast<long long>(p.B) * p.T, p.d,
                          p.row_bytes / 2, csa::kTileKeys, swz)) {
        return CSA_ERR_CUDA;
    }

    const KernelFn kern = pick_kernel(plan);
    // The kernel's warpgroups trade registers (setmaxnreg); that only adds up
    // when the kernel was built with exactly the launch count it assumes.
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess)
        return CSA_ERR_CUDA;
    if (fa.numRegs != csa::kLaunchRegs)
        return CSA_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, p.smem_bytes) !=
        cudaSuccess)
        return CSA_ERR_CUDA;
    const int sel_smem = static_cast<int>(sizeof(csa::SelSmem)) + 16;
    if (cudaFuncSetAttribute(csa::select_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             sel_smem) != cudaSuccess)
        return CSA_ERR_CUDA;
    const int sms = device_sms();
    int launched = 0;
    for (int qb_lo = 0; qb_lo < plan.nqb_total; qb_lo += plan.qb_chunk) {
        const int nqb = plan.nqb_total - qb_lo < plan.qb_chunk ? plan.nqb_total - qb_lo
                                                              : plan.qb_chunk;
        NvtxRange chunk_range("csa launch chunk: fused scoring + exact select");
        p.qb_lo = qb_lo;
        p.nqb = nqb;
        p.n_items = p.B * nqb * p.nsplit;
        const int grid = p.n_items < plan.grid ? p.n_items : plan.grid;
        if (!mark(launched++, stream))
            return CSA_ERR_CUDA;
        kern<<<grid, csa::kThreads, p.smem_bytes, stream>>>(tmQ, tmK, p);
        if (cudaGetLastError() != cudaSuccess)
            return CSA_ERR_CUDA;
        csa::SelParams sp;
        sp.lists = p.lists;
        sp.counts = p.counts;
        sp.rows = p.B * nqb * p.qps;
        sp.nsplit = p.nsplit;
        sp.cap = p.cap;
        sp.topk = p.topk;
        sp.B = p.B;
        sp.S = p.S;
        sp.qps = p.qps;
        sp.nqb = nqb;
        sp.qb_lo = qb_lo;
        sp.out_idx = a->out_idx;
        sp.out_score = a->out_score;
        const int sel_slots = csa::kSelCtasPerSm * sms;
        const int sel_grid = sp.rows < sel_slots ? sp.rows : sel_slots;
        if (!mark(launched++, stream))
            return CSA_ERR_CUDA;
        csa::select_topk_kernel<<<sel_grid, csa::kSelThreads, sel_smem, stream>>>(sp);
        if (cudaGetLastError() != cudaSuccess)
            return CSA_ERR_CUDA;
    }
    if (!mark(launched, stream))
        return CSA_ERR_CUDA;
    return CSA_OK;
}

} // namespace

extern "C" {

size_t csa_indexer_workspace_size(const csa_args_t *args)
{
    if (validate(args) != CSA_OK)
        return 0;
    if (static_cast<long long>(args->B) * args->S == 0 || args->T == 0)
        return 0;
    const int sms = device_sms();
    if (sms <= 0)
        return 0;
    Plan plan;
    if (make_plan(args, sms, kDefaultWorkspaceCap, &plan) != CSA_OK)
        return 0;
    return plan.ws_total;
}

csa_status_t csa_indexer_plan(const csa_args_t *args, csa_plan_t *out)
{
    if (!out)
        return CSA_ERR_INVALID_ARG;
    std::memset(out, 0, sizeof *out);
    csa_status_t st = validate(args);
    if (st != CSA_OK)
        return st;
    if (static_cast<long long>(args->B) * args->S == 0)
        return CSA_OK;
    if (args->T == 0) {
        out->launches = 1;
        return CSA_OK;
    }
    const int sms = device_sms();
    if (sms <= 0)
        return CSA_ERR_CUDA;
    Plan plan;
    st = make_plan(args, sms, kDefaultWorkspaceCap, &plan);
    if (st != CSA_OK)
        return st;
    out->grid = plan.grid;
    out->threads = csa::kThreads;
    out->smem_bytes = plan.p.smem_bytes;
    out->stages = plan.p.stages;
    out->queries_per_block = plan.p.qps;
    out->num_splits = plan.p.nsplit;
    out->launches = 2 * plan.chunks;
    out->workspace_bytes = plan.ws_total;
    return CSA_OK;
}

csa_status_t csa_indexer_topk_ex(const csa_args_t *args, void *workspace, size_t workspace_bytes,
                                 cudaStream_t stream)
{
    NvtxRange range("csa_indexer_topk_ex");
    csa_status_t st = validate(args);
    if (st != CSA_OK)
        return st;
    const long long rows = static_cast<long long>(args->B) * args->S;
    if (rows == 0)
        return CSA_OK;
    if (args->T == 0) {
        pad_outputs_kernel<<<256, 256, 0, stream>>>(args->out_idx, args->out_score,
                                                    rows * args->topk);
        return cudaGetLastError() == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
    }
    const int sms = device_sms();
    if (sms <= 0)
        return CSA_ERR_CUDA;
    Plan plan;
    st = make_plan(args, sms, kDefaultWorkspaceCap, &plan);
    if (st != CSA_OK)
        return st;
    if (workspace) {
        if (workspace_bytes < plan.ws_total)
            return CSA_ERR_WORKSPACE;
        if (!aligned(workspace, 256))
            return CSA_ERR_INVALID_ARG;
        return launch(args, plan, workspace, stream);
    }
    void *ws = nullptr;
    if (cudaMallocAsync(&ws, plan.ws_total, stream) != cudaSuccess)
        return CSA_ERR_CUDA;
    st = launch(args, plan, ws, stream);
    if (cudaFreeAsync(ws, stream) != cudaSuccess && st == CSA_OK)
        st = CSA_ERR_CUDA;
    return st;
}

csa_status_t csa_indexer_topk(const void *q, const float *w, const void *k, int B, int S, int T,
                              int H_I, int d, int m, int topk, int causal, int32_t *out_idx,
                              float *out_score, cudaStream_t stream)
{
    csa_args_t a;
    std::memset(&a, 0, sizeof a);
    a.q = q;
    a.w = w;
    a.k = k;
    a.k_scale = nullptr;
    a.B = B;
    a.S = S;
    a.T = T;
    a.H_I = H_I;
    a.d = d;
    a.m = m;
    a.topk = topk;
    a.causal = causal;
    a.key_dtype = CSA_KEY_BF16;
    a.mode = CSA_MODE_TOPK;
    a.q_offset = CSA_Q_OFFSET_DEFAULT;
    a.num_splits = 0;
    a.query_pieces = 0;
    a.out_idx = out_idx;
    a.out_score = out_score;
    return csa_indexer_topk_ex(&a, nullptr, 0, stream);
}

const char *csa_status_string(csa_status_t status)
{
    switch (status) {
    case CSA_OK: return "ok";
    case CSA_ERR_INVALID_ARG: return "invalid argument";
    case CSA_ERR_UNSUPPORTED: return "unsupported shape or option";
    case CSA_ERR_WORKSPACE: return "workspace too small";
    case CSA_ERR_CUDA: return "CUDA runtime error";
    case CSA_ERR_TIMEOUT: return "device-side wait timed out";
    case CSA_ERR_DEBUG_CHECK: return "debug-build index check failed on the device";
    }
    return "unknown status";
}

csa_status_t csa_last_device_error(cudaStream_t stream)
{
    if (cudaStreamSynchronize(stream) != cudaSuccess)
        return CSA_ERR_CUDA;
    int h[4] = {0, 0, 0, 0};
    if (cudaMemcpyFromSymbol(h, csa::g_csa_error, sizeof h) != cudaSuccess)
        return CSA_ERR_CUDA;
    if (h[0] == 0)
        return CSA_OK;
    const int zero[4] = {0, 0, 0, 0};
    if (cudaMemcpyToSymbol(csa::g_csa_error, zero, sizeof zero) != cudaSuccess)
        return CSA_ERR_CUDA;
    if (h[0] == csa::kErrTimeout)
        return CSA_ERR_TIMEOUT;
    return h[0] == csa::kErrDebugCheck ? CSA_ERR_DEBUG_CHECK : CSA_ERR_CUDA;
}

void csa_set_wait_limit(unsigned long long cycles)
{
    g_wait_limit = cycles ? cycles : kDefaultWaitLimit;
}

csa_status_t csa_set_launch_events(cudaEvent_t *events, int n)
{
    if (n < 0 || (n > 0 && !events))
        return CSA_ERR_INVALID_ARG;
    t_events = n > 0 ? events : nullptr;
    t_n_events = n;
    return CSA_OK;
}

int csa_version(void) { return kVersion; }

} // extern "C"

// ---------------------------------------------------------------------------
// Sparse attention over the selected keys.
namespace {

csa_status_t validate_attn(const csa_attn_args_t *a)
{
    if (!a)
        return CSA_ERR_INVALID_ARG;
    if (a->B < 0 || a->S < 0 || a->T < 0 || a->HA <= 0 || a->Dk <= 0 || a->Dv <= 0 ||
        a->topk <= 0 || a->ld_v < a->Dv || !(a->scale == a->scale))
        return CSA_ERR_INVALID_ARG;
    if (static_cast<long long>(a->B) * a->S == 0)
        return CSA_OK;
    if (!a->q || !a->idx || !a->out || (a->T > 0 && (!a->k || !a->v)))
        return CSA_ERR_INVALID_ARG;
    if (!aligned(a->q, 16) || (a->k && !aligned(a->k, 16)) || (a->v && !aligned(a->v, 16)) ||
        !aligned(a->idx, 4) || !aligned(a->out, 16) || (a->ld_v * 2) % 16 != 0)
        return CSA_ERR_INVALID_ARG;
    if (a->HA > csa::attn::kRows || a->Dk % 64 != 0 || a->Dk > 256 || a->Dv % 64 != 0 ||
        a->Dv > 256)
        return CSA_ERR_UNSUPPORTED;
    const long long rows_q = static_cast<long long>(a->B) * a->S * a->HA;
    if (rows_q + csa::attn::kRows >= (1ll << 31) || static_cast<long long>(a->B) * a->T >= (1ll << 31) ||
        static_cast<long long>(a->B) * a->S * a->topk >= (1ll << 40))
        return CSA_ERR_UNSUPPORTED;
    return CSA_OK;
}

__global__ void zero_kernel(float *x, long long n)
{
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<long long>(gridDim.x) * blockDim.x)
        x[i] = 0.0f;
}

} // namespace

extern "C" csa_status_t csa_sparse_attention(const csa_attn_args_t *args, cudaStream_t stream)
{
    NvtxRange range("csa_sparse_attention");
    const csa_status_t st = validate_attn(args);
    if (st != CSA_OK)
        return st;
    const long long rows = static_cast<long long>(args->B) * args->S;
    if (rows == 0)
        return CSA_OK;
    if (args->T == 0) {
        zero_kernel<<<256, 256, 0, stream>>>(args->out, rows * args->HA * args->Dv);
        return cudaGetLastError() == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
    }
    using namespace csa::attn;
    AttnParams p;
    std::memset(&p, 0, sizeof p);
    p.B = args->B;
    p.S = args->S;
    p.T = args->T;
    p.HA = args->HA;
    p.Dk = args->Dk;
    p.Dv = args->Dv;
    p.topk = args->topk;
    p.sl2 = args->scale * 1.4426950408889634f;
    p.idx = args->idx;
    p.out = args->out;
    p.wait_limit = static_cast<long long>(g_wait_limit);
    // shared memory: the query block, the key ring, the value ring, P,
    // barriers; two stages per ring where they fit, else one
    p.k_stage_bytes = kKeys * p.Dk * 2;
    p.v_stage_bytes = kKeys * p.Dv * 2;
    const int q_bytes = kRows * p.Dk * 2;
    const int p_bytes = kRows * kKeys * 2;
    const int fixed = q_bytes + p_bytes + static_cast<int>(sizeof(AttnBarriers)) + 64 + 1024;
    static const int kChoices[4][2] = {{2, 2}, {2, 1}, {1, 2}, {1, 1}};
    p.k_stages = 0;
    for (const auto &c : kChoices)
        if (fixed + c[0] * p.k_stage_bytes + c[1] * p.v_stage_bytes <= kSmemLimit) {
            p.k_stages = c[0];
            p.v_stages = c[1];
            break;
        }
    if (p.k_stages == 0)
        return CSA_ERR_UNSUPPORTED;
    p.off_q = 0;
    p.off_k = q_bytes;
    p.off_v = p.off_k + p.k_stages * p.k_stage_bytes;
    p.off_p = p.off_v + p.v_stages * p.v_stage_bytes;
    p.off_bar = p.off_p + p_bytes;
    int smem_bytes = p.off_bar + static_cast<int>(sizeof(AttnBarriers)) + 64 + 1024;
    // more than half of the SM: one CTA per SM, so its 512-column TMEM
    // allocation never waits on a neighbour
    if (smem_bytes < kSmemLimit / 2 + 1024)
        smem_bytes = kSmemLimit / 2 + 1024;

    p.k = static_cast<const uint8_t *>(args->k);
    p.v = static_cast<const uint8_t *>(args->v);
    p.v_row_bytes = args->ld_v * 2;
    CUtensorMap tmQ;
    const CUtensorMapDataType bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    // HA <= 64: the query block (64 rows) is loaded twice and the warp pairs
    // split each tile's keys; otherwise one 128-row block
    p.split = p.HA <= kRows / 2 ? 1 : 0;
    if (!make_tmap(&tmQ, bf, args->q, rows * p.HA, p.Dk, 64, p.split ? kRows / 2 : kRows,
                   CU_TENSOR_MAP_SWIZZLE_128B))
        return CSA_ERR_CUDA;
    // the warpgroups trade registers (setmaxnreg): only valid for a build
    // with exactly the launch count the split assumes
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, sparse_attn_kernel) != cudaSuccess)
        return CSA_ERR_CUDA;
    if (fa.numRegs != kLaunchRegs)
        return CSA_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(sparse_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem_bytes) != cudaSuccess)
        return CSA_ERR_CUDA;
    const int sms = device_sms();
    if (sms <= 0)
        return CSA_ERR_CUDA;
    const int grid = rows < sms ? static_cast<int>(rows) : sms;
    if (!mark(0, stream))
        return CSA_ERR_CUDA;
    sparse_attn_kernel<<<grid, kThreads, smem_bytes, stream>>>(tmQ, p);
    if (cudaGetLastError() != cudaSuccess)
        return CSA_ERR_CUDA;
    if (!mark(1, stream))
        return CSA_ERR_CUDA;
    return CSA_OK;
}

// ---------------------------------------------------------------------------
// Exact merge of top-k lists over disjoint key ranges (key shards).
namespace {

// One CTA per (row, list): the list's valid entries (index >= 0), in order,
// as 64-bit keys (score image << 32 | ~(index + offset)) in the select
// kernel's list layout, and their count.
__global__ void __launch_bounds__(256) pack_lists_kernel(csa::SelParams sp, const int32_t *const *idx,
                                                         const float *const *score,
                                                         const long long *offset, int k_in,
                                                         uint64_t *lists, int *counts)
{
    __shared__ int warp_tot[8];
    const int r = blockIdx.x / sp.nsplit, l = blockIdx.x % sp.nsplit;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int32_t *src_i = idx[l] + static_cast<size_t>(r) * k_in;
    const float *src_s = score[l] + static_cast<size_t>(r) * k_in;
    uint64_t *dst = lists + (static_cast<size_t>(r) * sp.nsplit + l) * sp.cap;
    int base = 0;
    for (int j0 = 0; j0 < k_in; j0 += 256) {
        const int j = j0 + tid;
        const int32_t s = j < k_in ? src_i[j] : -1;
        const bool ok = s >= 0;
        const uint32_t m = __ballot_sync(0xffffffffu, ok);
        if (lane == 0)
            warp_tot[wid] = __popc(m);
        __syncthreads();
        int before = 0, tot = 0;
        for (int w = 0; w < 8; ++w) {
            before += w < wid ? warp_tot[w] : 0;
            tot += warp_tot[w];
        }
        if (ok) {
            const long long g = static_cast<long long>(s) + offset[l];
            dst[base + before + __popc(m & ((1u << lane) - 1u))] =
                csa::make_key(csa::ord_of_score(src_s[j]), static_cast<uint32_t>(g));
        }
        base += tot;
        __syncthreads();
    }
    if (tid == 0)
        counts[static_cast<size_t>(r) * sp.nsplit + l] = base;
}

size_t merge_lists_bytes(int n_lists, int rows, int k_in)
{
    return align256(static_cast<size_t>(rows) * n_lists * k_in * 8);
}

size_t merge_ws_bytes(int n_lists, int rows, int k_in)
{
    return merge_lists_bytes(n_lists, rows, k_in) + align256(static_cast<size_t>(rows) * n_lists * 4) +
           align256(static_cast<size_t>(n_lists) * (2 * sizeof(void *) + sizeof(long long)));
}

} // namespace

extern "C" size_t csa_merge_workspace_size(int n_lists, int rows, int k_in)
{
    if (n_lists < 1 || n_lists > csa::kSelMaxSplits || rows < 0 || k_in < 1)
        return 0;
    return merge_ws_bytes(n_lists, rows, k_in);
}

extern "C" csa_status_t csa_merge_topk(const int32_t *const *idx, const float *const *score,
                                       const long long *key_offset, int n_lists, int rows,
                                       int k_in, int topk, int32_t *out_idx, float *out_score,
                                       void *workspace, size_t workspace_bytes,
                                       cudaStream_t stream)
{
    NvtxRange range("csa_merge_topk");
    if (!idx || !score || !key_offset || n_lists < 1 || n_lists > csa::kSelMaxSplits ||
        rows < 0 || k_in < 1 || topk < 1)
        return CSA_ERR_INVALID_ARG;
    if (topk > csa::kMaxTopk)
        return CSA_ERR_UNSUPPORTED;
    if (rows == 0)
        return CSA_OK;
    if (!out_idx || !out_score || !aligned(out_idx, 4) || !aligned(out_score, 4))
        return CSA_ERR_INVALID_ARG;
    for (int l = 0; l < n_lists; ++l) {
        if (!idx[l] || !score[l] || !aligned(idx[l], 4) || !aligned(score[l], 4) ||
            key_offset[l] < 0 || key_offset[l] + k_in >= (1ll << 31))
            return CSA_ERR_INVALID_ARG;
    }
    const size_t need = merge_ws_bytes(n_lists, rows, k_in);
    void *ws = workspace;
    if (ws) {
        if (workspace_bytes < need)
            return CSA_ERR_WORKSPACE;
        if (!aligned(ws, 256))
            return CSA_ERR_INVALID_ARG;
    } else if (cudaMallocAsync(&ws, need, stream) != cudaSuccess) {
        return CSA_ERR_CUDA;
    }
    // the list pointers and offsets go to the device through the workspace tail
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    uint64_t *lists = reinterpret_cast<uint64_t *>(w8);
    int *counts = reinterpret_cast<int *>(w8 + merge_lists_bytes(n_lists, rows, k_in));
    uint8_t *tail = w8 + merge_lists_bytes(n_lists, rows, k_in) +
                    align256(static_cast<size_t>(rows) * n_lists * 4);
    const int32_t **d_idx = reinterpret_cast<const int32_t **>(tail);
    const float **d_score = reinterpret_cast<const float **>(tail + n_lists * sizeof(void *));
    long long *d_off = reinterpret_cast<long long *>(tail + 2 * n_lists * sizeof(void *));
    csa_status_t st = CSA_OK;
    if (cudaMemcpyAsync(d_idx, idx, n_lists * sizeof(void *), cudaMemcpyHostToDevice, stream) !=
            cudaSuccess ||
        cudaMemcpyAsync(d_score, score, n_lists * sizeof(void *), cudaMemcpyHostToDevice, stream) !=
            cudaSuccess ||
        cudaMemcpyAsync(d_off, key_offset, n_lists * sizeof(long long), cudaMemcpyHostToDevice,
                        stream) != cudaSuccess)
        st = CSA_ERR_CUDA;
    csa::SelParams sp;
    std::memset(&sp, 0, sizeof sp);
    sp.lists = lists;
    sp.counts = counts;
    sp.rows = rows;
    sp.nsplit = n_lists;
    sp.cap = k_in;
    sp.topk = topk;
    sp.B = 1;
    sp.S = rows;
    sp.qps = 1;
    sp.nqb = rows;
    sp.qb_lo = 0;
    sp.out_idx = out_idx;
    sp.out_score = out_score;
    if (st == CSA_OK) {
        pack_lists_kernel<<<static_cast<unsigned>(rows) * n_lists, 256, 0, stream>>>(
            sp, d_idx, d_score, d_off, k_in, lists, counts);
        if (cudaGetLastError() != cudaSuccess)
            st = CSA_ERR_CUDA;
    }
    const int sel_smem = static_cast<int>(sizeof(csa::SelSmem)) + 16;
    if (st == CSA_OK && cudaFuncSetAttribute(csa::select_topk_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             sel_smem) != cudaSuccess)
        st = CSA_ERR_CUDA;
    const int sms = device_sms();
    if (st == CSA_OK && sms <= 0)
        st = CSA_ERR_CUDA;
    if (st == CSA_OK) {
        const int slots = csa::kSelCtasPerSm * sms;
        csa::select_topk_kernel<<<rows < slots ? rows : slots, csa::kSelThreads, sel_smem, stream>>>(sp);
        if (cudaGetLastError() != cudaSuccess)
            st = CSA_ERR_CUDA;
    }
    if (!workspace && cudaFreeAsync(ws, stream) != cudaSuccess && st == CSA_OK)
        st = CSA_ERR_CUDA;
    return st;
}

// ---------------------------------------------------------------------------
// OR-union of several layers' selections.
extern "C" csa_status_t csa_union_selections(const int32_t *const *lists, int n_lists, int rows,
                                             int topk, int T, int cap, int32_t *out,
                                             int32_t *count, cudaStream_t stream)
{
    NvtxRange range("csa_union_selections");
    using csa::uni::UnionParams;
    if (rows < 0 || topk <= 0 || T < 0 || cap <= 0 || n_lists < 1 ||
        n_lists > csa::uni::kMaxLists || !lists)
        return CSA_ERR_INVALID_ARG;
    if (rows == 0)
        return CSA_OK;
    if (!out || !count || !aligned(out, 4) || !aligned(count, 4))
        return CSA_ERR_INVALID_ARG;
    UnionParams p;
    std::memset(&p, 0, sizeof p);
    for (int l = 0; l < n_lists; ++l) {
        if (!lists[l] || !aligned(lists[l], 4))
            return CSA_ERR_INVALID_ARG;
        p.lists[l] = lists[l];
    }
    p.n_lists = n_lists;
    p.rows = rows;
    p.topk = topk;
    p.T = T;
    p.cap = cap;
    p.words = (T + 31) / 32;
    if (p.words < 1)
        p.words = 1;
    const long long smem = (static_cast<long long>(p.words) + csa::uni::kThreads / 32) * 4;
    if (smem > kSmemLimit)
        return CSA_ERR_UNSUPPORTED;
    p.out = out;
    p.count = count;
    if (cudaFuncSetAttribute(csa::uni::union_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return CSA_ERR_CUDA;
    const int sms = device_sms();
    if (sms <= 0)
        return CSA_ERR_CUDA;
    const int per_sm = smem > kSmemLimit / 2 ? 1 : (smem > kSmemLimit / 4 ? 2 : 4);
    const int grid = rows < per_sm * sms ? rows : per_sm * sms;
    csa::uni::union_kernel<<<grid, csa::uni::kThreads, static_cast<int>(smem), stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Allocation-free entry point.
//
// Some callers cannot allocate device memory at call time: serving loops that
// must not risk cudaMalloc's device-wide synchronisation in the middle of a
// latency-critical step, and hosts whose memory budget is fixed up front and
// that forbid allocations outside their own pool.  For them the scratch this
// operation needs lives in one fixed array below, created with the library's
// module on every GPU that loads it and held until the process exits.
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20; // 64 MiB

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
void *g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once
// per device (host code cannot use the array's name as a device pointer).
csa_status_t noalloc_scratch(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return CSA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p)
            return CSA_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return CSA_OK;
}

} // namespace

extern "C" csa_status_t csa_indexer_topk_noalloc(const csa_args_t *args, cudaStream_t stream)
{
    NvtxRange range("csa_indexer_topk_noalloc");
    csa_status_t st = validate(args);
    if (st != CSA_OK)
        return st;
    const long long rows = static_cast<long long>(args->B) * args->S;
    if (rows == 0)
        return CSA_OK;
    if (args->T == 0) {
        pad_outputs_kernel<<<256, 256, 0, stream>>>(args->out_idx, args->out_score,
                                                    rows * args->topk);
        return cudaGetLastError() == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
    }
    const int sms = device_sms();
    if (sms <= 0)
        return CSA_ERR_CUDA;
    // The candidate lists scale with the number of query blocks in flight:
    // the plan runs as many launch chunks as the fixed scratch requires.
    Plan plan;
    st = make_plan(args, sms, kNoAllocScratchBytes, &plan);
    if (st != CSA_OK)
        return st;
    void *scratch = nullptr;
    st = noalloc_scratch(&scratch);
    if (st != CSA_OK)
        return st;
    return launch(args, plan, scratch, stream);
}

#ifdef CSA_PROFILE
// Profiling build only: per-CTA role counters of the last launches.
extern "C" int csa_profile_read(unsigned long long *out, int n)
{
    const size_t bytes = sizeof(unsigned long long) * csa::kProfCtas * 32;
    if (n * sizeof(unsigned long long) < bytes)
        return -1;
    return cudaMemcpyFromSymbol(out, csa::g_csa_prof, bytes) == cudaSuccess ? 0 : -1;
}

extern "C" int csa_profile_reset(void)
{
    static unsigned long long zero[csa::kProfCtas][32];
    return cudaMemcpyToSymbol(csa::g_csa_prof, zero, sizeof zero) == cudaSuccess ? 0 : -1;
}
#endif
