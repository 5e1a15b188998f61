/*
 * csa_indexer.h -- C ABI of the B200 (sm_100a) CSA lightning-indexer top-k.
 *
 * The operation ("StreamIndex: Memory-Bounded Compressed Sparse Attention via
 * Streaming Top-k", abstract: a lightning indexer scores compressed keys, the
 * top-k are selected per query, and the full [B,S,H_I,T] score tensor is
 * never materialised):
 *
 *   for every batch b and query row i, with absolute position t = i + q_offset,
 *     key s (covering tokens [s*m, (s+1)*m)) is visible iff !causal or
 *     (s+1)*m - 1 <= t, and
 *       I[t,s] = sum_h w[b,i,h] * ReLU( sum_j q[b,i,h,j] * k[b,s,j] )
 *     (FP8 keys: k[b,s,j] = k_scale[b,s] * E4M3(k8[b,s,j]))
 *   CSA_MODE_TOPK: return the min(topk, #visible) visible keys with the
 *     largest I, ordered by I descending, equal scores by ascending s.
 *   CSA_MODE_GATE: keep only visible keys with sigmoid(I) > 0.5, i.e. I > 0
 *     ("FlashMemory-DeepSeek-V4: Lightning Index Ultra-Long Context via
 *     Lookahead Sparse Attention", "What carries the argument": a sigmoid
 *     gate with a fixed 0.5 threshold in place of a fixed top-k), at most
 *     topk of them, chosen and ordered as in CSA_MODE_TOPK.
 *   Unused output slots hold index -1 and score -inf.  A zero score is +0.0.
 *
 * Layouts (all contiguous, row-major, DEVICE memory owned by the caller):
 *   q         [B, S, H_I, d]  bfloat16
 *   w         [B, S, H_I]     float32
 *   k         [B, T, d]       bfloat16 (CSA_KEY_BF16) or E4M3 bytes (CSA_KEY_E4M3)
 *   k_scale   [B, T]          float32, > 0 (CSA_KEY_E4M3 only)
 *   out_idx   [B, S, topk]    int32, key indices in [0, T) or -1
 *   out_score [B, S, topk]    float32
 * q and k must be 16-byte aligned (the tensor-memory copies read them);
 * w, k_scale, out_idx and out_score 4-byte aligned.  Inputs must be finite;
 * NaN or Inf inputs give unspecified (but memory-safe) results.
 *
 * Arithmetic: products q.k accumulate in fp32 on the tensor cores, the head
 * sum in fp32.  With E4M3 keys the key bytes are multiplied as stored and each
 * query row (one (query, head) pair) is carried as sigma * (hi8 + lo8), two
 * E4M3 pieces with a power-of-two sigma: exact for every element of at least
 * 2^-9 of the row's largest |q|, within 2^-17 of that largest otherwise.
 *
 * Supported shapes: H_I a power of two in [1, 256]; d in {32, 64, 128};
 * 1 <= topk <= 2048; m >= 1; T, S < 2^31.  Anything else returns
 * CSA_ERR_UNSUPPORTED before any launch.  There is no CPU fallback.
 *
 * All calls are stream-ordered on `stream`: they enqueue work and return
 * without synchronising.  Errors are returned as status codes; no call throws
 * across this boundary.  Arguments are validated before any launch
 * (CSA_ERR_INVALID_ARG / CSA_ERR_UNSUPPORTED leave the outputs untouched).
 * Every device-side wait is bounded; a wait that runs out records a timeout
 * that csa_last_device_error() reports, and the kernel exits cleanly.
 */
#ifndef CSA_INDEXER_H
#define CSA_INDEXER_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    CSA_OK = 0,
    CSA_ERR_INVALID_ARG = 1, /* null pointer, negative size, bad enum, misaligned pointer */
    CSA_ERR_UNSUPPORTED = 2, /* valid but outside the supported shapes listed above       */
    CSA_ERR_WORKSPACE = 3,   /* caller workspace smaller than csa_indexer_workspace_size  */
    CSA_ERR_CUDA = 4,        /* a CUDA runtime call failed (launch, allocation, ...)      */
    CSA_ERR_TIMEOUT = 5,     /* a bounded device-side wait ran out (see csa_last_device_error) */
    CSA_ERR_DEBUG_CHECK = 6  /* debug build (-DCSA_DEBUG) only: a kernel's shared-memory,
                                tensor-memory, buffer or output index failed its bounds
                                check; the access was skipped (csa_last_device_error) */
} csa_status_t;

typedef enum { CSA_KEY_BF16 = 0, CSA_KEY_E4M3 = 1 } csa_key_dtype_t;

/* q_offset value that selects the default alignment max(0, T*m - S). */
#define CSA_Q_OFFSET_DEFAULT (-9223372036854775807LL - 1)
typedef enum { CSA_MODE_TOPK = 0, CSA_MODE_GATE = 1 } csa_mode_t;

/* Full argument set of one indexer call.  Pointers are device pointers. */
typedef struct {
    const void *q;         /* [B,S,H_I,d] bf16                                 */
    const float *w;        /* [B,S,H_I] fp32                                   */
    const void *k;         /* [B,T,d] bf16 or E4M3 bytes                       */
    const float *k_scale;  /* [B,T] fp32 > 0 for CSA_KEY_E4M3, else NULL       */
    int B, S, T, H_I, d, m, topk;
    int causal;            /* 0: every key visible; 1: the causal rule above   */
    int key_dtype;         /* csa_key_dtype_t                                  */
    int mode;              /* csa_mode_t                                       */
    long long q_offset;    /* absolute position of query row 0 (may be
                              negative: rows before position 0 see no key);
                              CSA_Q_OFFSET_DEFAULT selects max(0, T*m - S)
                              (queries end where the keys' token span ends)  */
    int num_splits;        /* key-range splits per query block; 0 = automatic  */
    int32_t *out_idx;      /* [B,S,topk]                                       */
    float *out_score;      /* [B,S,topk]                                       */
    int query_pieces;      /* E4M3 keys only: how each bf16 query row meets the
                              E4M3 keys on the tensor core.  0 or 2 (default):
                              as sigma*(hi8 + lo8), two E4M3 pieces (exact for
                              every element of at least 2^-9 of the row's
                              largest |q|).  1: as sigma*hi8, one E4M3 rounding
                              per element (relative error up to 2^-4): half the
                              tensor work, at a cost in recall.  Must be 0 with
                              bf16 keys.                                         */
} csa_args_t;

/*
 * The plain entry point: bf16 q and k, ReLU top-k, default q_offset.
 * Needs scratch memory, which it takes with cudaMallocAsync on `stream` and
 * returns with cudaFreeAsync on the same stream (stream-ordered; no sync).
 */
csa_status_t csa_indexer_topk(const void *q, const float *w, const void *k,
                              int B, int S, int T, int H_I, int d, int m, int topk,
                              int causal, int32_t *out_idx, float *out_score,
                              cudaStream_t stream);

/*
 * Bytes of device scratch csa_indexer_topk_ex needs for these arguments
 * (depends on shapes, topk and the device's SM count, not on the data).
 * Returns 0 for arguments that csa_indexer_topk_ex would reject.
 */
size_t csa_indexer_workspace_size(const csa_args_t *args);

/*
 * Extended entry point: any key dtype and mode, explicit q_offset and split
 * count.  `workspace` is caller-owned device memory of at least
 * csa_indexer_workspace_size(args) bytes, 256-byte aligned, used only for
 * the duration of the enqueued work; pass NULL to have the call allocate and
 * free it stream-ordered on `stream` (cudaMallocAsync/cudaFreeAsync).
 * Two calls that share a workspace must not overlap on the GPU.
 */
csa_status_t csa_indexer_topk_ex(const csa_args_t *args, void *workspace,
                                 size_t workspace_bytes, cudaStream_t stream);

/*
 * Same operation as csa_indexer_topk_ex, for callers that cannot allocate
 * device memory while they run: latency-critical serving loops that must not
 * risk cudaMalloc's device-wide synchronisation mid-step, and hosts whose
 * memory budget is fixed up front and that forbid allocations outside their
 * own pool.  The paper has no counterpart; this is a deployment variant.
 *
 * The call allocates nothing.  Its scratch is one fixed 64 MiB device array
 * inside this library (CSA_NOALLOC_SCRATCH_BYTES); a GPU holds it from the
 * library's first use on that device (at the latest the first call of this
 * entry point there) until the process exits.  The caller still passes all
 * inputs and outputs.  The first call on each device looks up that array's
 * device address (cudaGetSymbolAddress); make that first call before any
 * stream capture.  The scratch holds the kernels' per-CTA score buffers and
 * the candidate lists of the queries in flight (B * queries-per-block * splits
 * lists of topk + max(256, topk/4) 8-byte keys per block of queries); when all
 * of them do not fit, the call runs as several launch chunks of query blocks
 * (and fewer CTAs when the score buffers alone would not fit).  If one query
 * block of every sequence already needs more than the array (very large
 * B * topk), it returns CSA_ERR_WORKSPACE and launches nothing.  All calls
 * share the one array and nothing in it needs to start at zero, but two calls
 * that overlap on the GPU (different streams, or different host threads) race
 * on it and give undefined results: serialise them.
 */
#define CSA_NOALLOC_SCRATCH_BYTES (64ull << 20)
csa_status_t csa_indexer_topk_noalloc(const csa_args_t *args, cudaStream_t stream);

/*
 * Sparse attention over the selected keys: the step that consumes the
 * indexer's output ("StreamIndex: Memory-Bounded Compressed Sparse Attention
 * via Streaming Top-k", abstract: a sparse attention kernel reads only the
 * selected compressed keys).  For every batch b, query row i and head g < HA:
 *
 *   J = the entries of idx[b,i,0..topk) that lie in [0, T), in slot order
 *       (the indexer lists its selection first and pads with -1; an entry
 *       outside [0, T) is padding wherever it stands, and the slots after the
 *       last key are not read twice)
 *   out[b,i,g,:] = sum_j softmax_j( scale * q[b,i,g,:] . k[b,J_j,:] ) * v[b,J_j,:]
 *   (zeros when n = 0)
 *
 * One compressed cache row per key is shared by all heads.  Layouts (DEVICE
 * memory owned by the caller, row-major):
 *   q    [B, S, HA, Dk]  bfloat16, 16-byte aligned
 *   k    [B, T, Dk]      bfloat16, 16-byte aligned
 *   v    value row s of batch b at v + (b*T + s) * ld_v elements (bfloat16,
 *        16-byte aligned, ld_v >= Dv and ld_v * 2 a multiple of 16); v = k
 *        with ld_v = Dk reads the values as the first Dv elements of each key
 *        row (a latent cache)
 *   idx  [B, S, topk]    int32 (the indexer's out_idx)
 *   out  [B, S, HA, Dv]  float32, 16-byte aligned
 * Arithmetic: q.k on the tensor cores (bf16, fp32 accumulate), softmax in
 * fp32 (exp2 domain), the probabilities rounded to bf16 for P.V (fp32
 * accumulate).  Supported: 1 <= HA <= 128; Dk, Dv multiples of 64 up to 256.
 * Stream-ordered; status codes as above; no allocation.
 */
typedef struct {
    const void *q;
    const void *k;
    const void *v;
    long long ld_v;
    const int32_t *idx;
    int B, S, T, HA, Dk, Dv, topk;
    float scale;
    float *out;
} csa_attn_args_t;

csa_status_t csa_sparse_attention(const csa_attn_args_t *args, cudaStream_t stream);

/*
 * Exact merge of top-k lists made over disjoint key ranges, e.g. one list per
 * GPU when the keys are sharded across GPUs ("Million-Token Memory Without
 * the Global Bottleneck": keys split across GPUs, a selection on each, then
 * a combination that covers the global top).  idx and score are HOST arrays
 * of n_lists (1..64) DEVICE pointers, each [rows, k_in] (an indexer's
 * out_idx / out_score over its key range); key_offset is a HOST array of
 * n_lists offsets added to each list's indices (the first key of its range),
 * and entries with index < 0 are padding.  out_idx / out_score [rows, topk]
 * receive the topk largest scores of the union, ordered by score descending,
 * equal scores by ascending (offset) index, padded with -1 / -inf.  When
 * every list holds its range's top min(topk, k_in) keys with k_in >= topk,
 * this is exactly the top-k over all ranges.  workspace: device memory of
 * csa_merge_workspace_size(n_lists, rows, k_in) bytes, 256-byte aligned, or
 * NULL to allocate stream-ordered.  topk <= 2048.
 */
csa_status_t csa_merge_topk(const int32_t *const *idx, const float *const *score,
                            const long long *key_offset, int n_lists, int rows, int k_in,
                            int topk, int32_t *out_idx, float *out_score, void *workspace,
                            size_t workspace_bytes, cudaStream_t stream);
size_t csa_merge_workspace_size(int n_lists, int rows, int k_in);

/*
 * OR-union of several layers' selections ("FlashMemory-DeepSeek-V4:
 * Lightning Index Ultra-Long Context via Lookahead Sparse Attention", "What
 * carries the argument": the gated decisions of a few layers are combined by
 * OR-union).  lists is a HOST array of n_lists (1..8) DEVICE pointers, each
 * [rows, topk] int32 (an indexer's out_idx; entries outside [0, T) are
 * padding).  For every row, out[row, 0..count) receives the distinct keys any
 * list holds, in ascending key order, at most cap of them (the smallest keys
 * when the union is larger; size cap = n_lists * topk to keep every key), and
 * out[row, count..cap) is -1.  out [rows, cap] and count [rows] are device
 * int32, 4-byte aligned.  T up to about 1.8 million keys (a bitmap of the
 * row's keys in shared memory); larger returns CSA_ERR_UNSUPPORTED.
 * Stream-ordered; no allocation.
 */
csa_status_t csa_union_selections(const int32_t *const *lists, int n_lists, int rows, int topk,
                                  int T, int cap, int32_t *out, int32_t *count,
                                  cudaStream_t stream);

/* How csa_indexer_topk_ex would run a call (for benchmarks and tests). */
typedef struct {
    int grid;              /* CTAs of the fused kernel (persistent, <= SM count) */
    int threads;           /* threads per CTA                                    */
    int smem_bytes;        /* dynamic shared memory per CTA                      */
    int stages;            /* key-tile pipeline depth                            */
    int queries_per_block; /* queries one work item covers                       */
    int num_splits;        /* key-range splits per query block                   */
    int launches;          /* kernel launches per call: per launch chunk the      *
                            * fused scoring/filter kernel and the exact top-k   *
                            * select (0 or 1 for the empty cases)               */
    size_t workspace_bytes;
} csa_plan_t;

/*
 * Fills *plan for these arguments on the current device without launching
 * anything.  Returns the status csa_indexer_topk_ex would return before
 * launching (CSA_OK, CSA_ERR_INVALID_ARG, CSA_ERR_UNSUPPORTED, CSA_ERR_CUDA
 * when no device is present).  For B*S == 0 or T == 0 the plan is all zeros
 * apart from `launches` (0 or 1).
 */
csa_status_t csa_indexer_plan(const csa_args_t *args, csa_plan_t *plan);

/* Static text for a status code. */
const char *csa_status_string(csa_status_t status);

/*
 * Synchronises `stream`, then reports (and clears) the device error word that
 * bounded waits set when they run out on the current device, and that the
 * debug build's index checks set when one fails: CSA_OK, CSA_ERR_TIMEOUT,
 * CSA_ERR_DEBUG_CHECK, or CSA_ERR_CUDA if the synchronisation failed.
 */
csa_status_t csa_last_device_error(cudaStream_t stream);

/*
 * Cycle budget of every bounded device-side wait for later launches from this
 * process (default 4e9 cycles, about two seconds at the B200's clocks).
 * Tests shrink it to make a wait run out on purpose.  0 restores the default.
 */
void csa_set_wait_limit(unsigned long long cycles);

/*
 * Measurement hook (no counterpart in the pages): while set, every later call
 * on this host thread records events[j] on its stream immediately before its
 * j-th kernel launch and events[L] after its last one (L = launches of the
 * call), for j < n; events beyond n are not recorded.  For a single-chunk
 * plan the fused kernel runs between events[0] and events[1] and the top-k
 * select between events[1] and events[2].  The caller owns the events
 * (created with timing enabled) and keeps them alive while set; pass
 * (NULL, 0) to stop.  Returns CSA_ERR_INVALID_ARG for n < 0 or a NULL array
 * with n > 0.
 */
csa_status_t csa_set_launch_events(cudaEvent_t *events, int n);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int csa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* CSA_INDEXER_H */
