/*
 * li.h -- C ABI of libli, a B200 (sm_100a) LightningIndexer.
 *
 * The operation (mindspore.ops.lightning_indexer page, ".. math::"; CANN
 * LightningIndexerV2 guide, "三步计算流程"; VllmQuantLightningIndexer README,
 * "功能说明"): for every query token and every key it may see,
 *
 *     s(t) = sum_h W[h] * ReLU( [Scale_Q[h] * Scale_K[t] *] (q_h . k_t) )
 *
 * then the sparse_count keys with the largest s (ties: lower key index first)
 * are returned as int32 indices, optionally with their fp32 scores.
 *
 * Conventions shared by every entry point:
 *   - The caller owns all memory.  Every tensor pointer is a DEVICE pointer to
 *     a contiguous tensor (PA key blocks may be strided, see key_block_stride),
 *     16-byte aligned.  The library allocates nothing and never synchronises
 *     the stream, except li_read_device_status, which says so.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Every launch is asynchronous on it.
 *   - A return value other than LI_OK means that nothing was launched; the
 *     reason is in li_last_error() (a thread-local string).
 *   - Errors that only the device can see (an actual length beyond the tensor
 *     or the declared bound, a block id outside the pool, a negative dequant
 *     scale, a bounded wait that expired) never fault: the kernels clamp or
 *     skip the access and OR a bit into the status word at the start of the
 *     workspace.  Read it with li_read_device_status.
 */
#ifndef LI_H
#define LI_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LI_API __attribute__((visibility("default")))
#else
#define LI_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LI_OK = 0,
    LI_ERR_NULL = 1,         /* a required pointer is NULL                        */
    LI_ERR_SHAPE = 2,        /* a dimension or attribute is out of range          */
    LI_ERR_DTYPE = 3,        /* dtype combination not allowed                     */
    LI_ERR_LAYOUT = 4,       /* layout combination not allowed                    */
    LI_ERR_UNSUPPORTED = 5,  /* allowed by the pages but not built here           */
    LI_ERR_WORKSPACE = 6,    /* workspace missing, too small or misaligned        */
    LI_ERR_CUDA = 7,         /* a CUDA runtime call failed                        */
    LI_ERR_DEVICE = 8        /* li_read_device_status: the device flagged a problem */
} li_status;

typedef enum { LI_BF16 = 0, LI_FP16 = 1, LI_FP32 = 2, LI_FP8_E4M3 = 3, LI_INT8 = 4 } li_dtype;
typedef enum { LI_BSND = 0, LI_TND = 1, LI_PA_BSND = 2 } li_layout;

/* Bits of the device status word (li_read_device_status). */
#define LI_DEV_BAD_QLEN      0x01  /* query length / prefix sum out of range (clamped)  */
#define LI_DEV_BAD_KLEN      0x02  /* key length / prefix sum out of range (clamped)    */
#define LI_DEV_BAD_BLOCK     0x04  /* block_table entry outside [0, num_blocks) (skipped) */
#define LI_DEV_NEG_SCALE     0x08  /* negative dequant scale (the fold needs scales >= 0) */
#define LI_DEV_TIMEOUT       0x10  /* a bounded pipeline wait expired                   */

/*
 * Op attributes and dimensions (mindspore page, "参数" / "关键字参数"; CANN
 * guide, "约束说明"; README, "参数说明").
 *   layout_q       LI_BSND: query [B,S1,N1,D], weights [B,S1,N1]
 *                  LI_TND : query [T1,N1,D],   weights [T1,N1]
 *   layout_k       LI_BSND: key [B,S2,N2,D]; LI_TND: key [T2,N2,D];
 *                  LI_PA_BSND: key [num_blocks,block_size,N2,D] addressed via block_table.
 *                  Without PA, layout_k must equal layout_q.
 *   dtype_qk       LI_BF16 / LI_FP16 (li_indexer); LI_FP8_E4M3 / LI_INT8 (li_quant_indexer)
 *   dtype_w        LI_BF16 / LI_FP16 / LI_FP32
 *   dtype_scale    LI_FP32 / LI_FP16 (li_quant_indexer only)
 *   N1             query heads, 1..64;  N2 key heads, must be 1
 *   D              head dim: 128, or 64 for 16-bit q/k (the TileLang test shape)
 *   num_blocks, block_size, max_blocks_per_seq
 *                  PA pool geometry; block_size a multiple of 16 in [16, 1024]
 *   key_block_stride  elements between consecutive PA blocks (0 = dense
 *                  block_size*N2*D); lets axis 0 of the pool be non-contiguous
 *   sparse_count   k, 1..8192 (CANN guide, "约束说明")
 *   sparse_mode    0 = every key inside the actual length; 3 = right-down causal:
 *                  key t is visible to query i of batch b iff t <= i + Sk_b - Sq_b
 *   pre_tokens, next_tokens  reserved; must be INT64_MAX
 *   return_value   1 = also write sparse_values (fp32)
 *   max_seqlen_k   host-side upper bound on every actual key length (0 = S2 for
 *                  BSND, T2 for TND, max_blocks_per_seq*block_size for PA).  It
 *                  sizes the workspace; longer actual lengths are clamped and flagged.
 *   init_num, local_num  sink tokens and local window (the MT lightning_indexer
 *                  attributes of the open-sourcing issue): the first init_num and
 *                  the last local_num visible keys of every row are always
 *                  selected, the best other visible keys fill the remaining
 *                  slots, all ordered by score.  0 = off; init_num + local_num
 *                  must not exceed sparse_count.
 *   cmp_ratio      compressed keys (CANN LightningIndexerV2 guide): every key
 *                  stands for cmp_ratio original tokens; 0 or 1 = none; a power
 *                  of two up to 128.  Indices count compressed keys.
 *   cmp_residual_k device int32 [B]: original key tokens left over after the
 *                  last whole compressed key, each < cmp_ratio.  Required when
 *                  cmp_ratio > 1 and sparse_mode == 3 (then a key is visible once
 *                  all of its original tokens are: key t is visible to query i iff
 *                  (t+1)*cmp_ratio - 1 <= i + Sk*cmp_ratio + residual - Sq);
 *                  ignored otherwise.  A residual outside [0, cmp_ratio) is
 *                  clamped and flagged with LI_DEV_BAD_KLEN.
 *   reserved       must be 0
 */
typedef struct {
    int32_t layout_q, layout_k;
    int32_t dtype_qk, dtype_w, dtype_scale;
    int32_t B, S1, S2, T1, T2, N1, N2, D;
    int32_t num_blocks, block_size, max_blocks_per_seq;
    int64_t key_block_stride;
    int32_t sparse_count, sparse_mode;
    int64_t pre_tokens, next_tokens;
    int32_t return_value;
    int32_t max_seqlen_k;
    int32_t init_num, local_num;
    int32_t cmp_ratio;
    int32_t reserved;
    const int32_t *cmp_residual_k;
} li_params;

/*
 * Output shape (CANN guide, "输出 shape 的推导依据"; mindspore page, "返回").
 * BSND query: sparse_indices is [B, S1, N2, k] (ndim 4); TND: [T1, N2, k]
 * (ndim 3).  sparse_values has the same shape when return_value is set.
 * out_dims must hold 4 entries.  Host only; validates params.
 */
LI_API li_status li_output_shape(const li_params *p, int64_t out_dims[4], int32_t *ndim);

/* Bytes of device workspace that li_indexer / li_quant_indexer need for `p`
 * (status word, scheduler tables and one fp32 score row per query).  Host only. */
LI_API li_status li_workspace_size(const li_params *p, size_t *bytes);

/*
 * The indexer on 16-bit query/key (mindspore page, whole signature; CANN guide,
 * "函数原型").
 *   query, key, weights   device tensors in the layouts above
 *   act_seq_q  int32 [B]: per-batch query lengths for BSND (NULL = S1 each), or
 *              prefix sums without a leading 0 for TND (required)
 *   act_seq_k  int32 [B]: per-batch key lengths for BSND (NULL = S2 each) and
 *              PA (required), or prefix sums for TND (required)
 *   block_table int32 [B, max_blocks_per_seq], PA only: physical block of each
 *              logical key block
 *   sparse_indices  int32 [rows, k] output; slots past min(k, visible) are -1
 *   sparse_values   fp32 [rows, k] output (NULL iff return_value == 0); padding -inf
 *   workspace       device buffer of li_workspace_size bytes, 256-byte aligned;
 *                   it must not be shared by calls that may run concurrently
 */
LI_API li_status li_indexer(const li_params *p, const void *query, const void *key, const void *weights,
                     const int32_t *act_seq_q, const int32_t *act_seq_k,
                     const int32_t *block_table, int32_t *sparse_indices, float *sparse_values,
                     void *workspace, size_t workspace_bytes, void *stream);

/*
 * The quantised indexer (VllmQuantLightningIndexer README, "功能说明" and
 * "参数说明"): q/k are fp8 e4m3 or int8, and the per-token-head dequant
 * scales multiply the dot product before the ReLU.  int8 q/k accumulate
 * exactly in s32 (|q.k| <= 2^21 for D = 128) and are converted to fp32.
 *   q_scale  dtype_scale (fp32 or fp16), same layout as weights ([B,S1,N1] or [T1,N1])
 *   k_scale  dtype_scale per key token: [B,S2,N2], [T2,N2] or [num_blocks,block_size,N2]
 * Scales must be >= 0 (then ReLU(sq*sk*x) = sq*sk*ReLU(x), which the kernel
 * uses); a negative scale is flagged with LI_DEV_NEG_SCALE.  Other arguments
 * as li_indexer.
 */
LI_API li_status li_quant_indexer(const li_params *p, const void *query, const void *key,
                           const void *weights, const void *q_scale, const void *k_scale,
                           const int32_t *act_seq_q, const int32_t *act_seq_k,
                           const int32_t *block_table, int32_t *sparse_indices,
                           float *sparse_values, void *workspace, size_t workspace_bytes,
                           void *stream);

/*
 * The Top-k stage on its own (CANN guide, "三步计算流程" step 3, with the
 * deterministic ordering of "确定性计算"): for each of `rows` fp32 score rows
 * (row r starts at scores + r*ld and its first row_len[r] entries are the
 * candidates; row_len NULL = ld for every row), write the k largest as
 * (index, value) pairs ordered by value descending, ties by lower index; pad
 * with -1 / -inf.  -0.0 counts as +0.0.  ld must be a multiple of 4.
 * sparse_values may be NULL.  Needs no workspace.
 */
LI_API li_status li_topk(const float *scores, int64_t ld, const int32_t *row_len, int32_t rows,
                  int32_t k, int32_t *sparse_indices, float *sparse_values, void *stream);

/*
 * li_indexer for callers that cannot hand the library any device memory of
 * their own.  The pages have no counterpart to it; it is an addition of this
 * library.
 *
 * Some callers cannot allocate device memory: an operator interface that
 * passes a kernel only its input and output tensors and has no workspace
 * mechanism, or a serving loop that keeps cudaMalloc off its hot path (the
 * call can synchronise the device and fragment a pre-reserved pool).  This
 * entry point takes the same arguments as li_indexer minus the workspace and
 * uses instead a scratch array of LI_NOALLOC_SCRATCH_BYTES compiled into the
 * library: every GPU that loads the library holds that memory until the
 * process exits.  It calls no allocator itself.
 *
 *   - Problems whose li_workspace_size exceeds LI_NOALLOC_SCRATCH_BYTES are
 *     rejected with LI_ERR_WORKSPACE before anything is launched; use
 *     li_indexer with a workspace for them.
 *   - The first call on a device looks up that device's copy of the array
 *     (cudaGetSymbolAddress); make that first call before any stream capture.
 *     The address belongs to the device's current context: a call made after
 *     that context was destroyed and re-created (cudaDeviceReset) looks it up
 *     again, so that call too should come before any capture.
 *   - All calls on a device share the one array and it keeps the contents of
 *     the last call.  Nothing in it has to start at zero (each call's
 *     scheduler overwrites the status and tables, and every score is written
 *     before it is read), but calls that may overlap on the GPU -- concurrent
 *     streams, or threads launching at the same time -- race on it.
 *   - The device status word of these calls sits in the library's scratch
 *     and is not exposed; use li_indexer with a workspace when the LI_DEV_*
 *     bits are needed.
 */
#define LI_NOALLOC_SCRATCH_BYTES (32u << 20)
LI_API li_status li_indexer_noalloc(const li_params *p, const void *query, const void *key,
                                    const void *weights, const int32_t *act_seq_q,
                                    const int32_t *act_seq_k, const int32_t *block_table,
                                    int32_t *sparse_indices, float *sparse_values, void *stream);

/*
 * Sparse attention over the selected keys: the consumer of the indexer's
 * output (CANN TileLang LightningIndexer guide, section "LightningIndexer 在
 * 稀疏注意力中的地位": an explicit index tensor names, for every query token,
 * the key/value subset it attends to, so attention costs O(N*S) instead of
 * O(N^2); the open-sourcing issue, section 3: the forward's sparse_indices feed
 * Sparse FlashAttention).  The pages give no formula of their own for it; this
 * library computes scaled dot-product attention restricted to each row's
 * selected keys, with one key/value head shared by all query heads:
 *
 *     J      = entries j of the row's index list with 0 <= j < Sk_b
 *     out_h  = sum_{j in J} softmax_j(scale * q_h . k_j) * v_j
 *     lse_h  = log sum_{j in J} exp(scale * q_h . k_j)
 *
 * and out = 0, lse = -inf for rows with J empty and for BSND padding rows.
 *
 *   layout_q       LI_BSND: query/out [B,S1,N1,D]; LI_TND: [T1,N1,D]
 *   layout_kv      LI_BSND: key [B,S2,1,D], value [B,S2,1,Dv]; LI_TND: [T2,1,D] /
 *                  [T2,1,Dv]; LI_PA_BSND: [num_blocks,block_size,1,D] / [..,Dv]
 *                  through block_table (a dense pool)
 *   dtype          LI_BF16 or LI_FP16 for query, key, value and out
 *   N1             query heads: 16, 32, 64 or 128
 *   D, Dv          128 and 128
 *   sparse_count   K, entries per index row, 1..65536
 *   softmax_scale  > 0 and finite (1/sqrt(D) is the usual choice)
 *   B, S1, S2, T1, T2, num_blocks, block_size, max_blocks_per_seq  as in li_params
 *   reserved       must be 0
 *
 *   sparse_indices int32 [rows, K] (the indexer's output layout): batch-local
 *                  key positions; -1 marks an empty slot.  An entry >= Sk_b or
 *                  below -1 is skipped and flagged with LI_DEV_BAD_INDEX.
 *   act_seq_q, act_seq_k, block_table   as for li_indexer
 *   out            [rows, N1, Dv] in dtype (device)
 *   lse            fp32 [rows, N1] (device) or NULL
 *   status         device int32 that receives LI_DEV_* bits by atomic OR, or
 *                  NULL; the caller clears it.  LI_DEV_BAD_INDEX: an entry
 *                  outside [-1, Sk_b) (skipped); LI_DEV_BAD_BLOCK: a
 *                  block_table entry outside [0, num_blocks) behind a valid
 *                  index (skipped); LI_DEV_TIMEOUT: a pipeline wait expired
 *                  (out and lse are then undefined; the kernel still ends)
 * Pointers: query, key, value and out 16-byte aligned; sparse_indices, lse and
 * status 4-byte aligned (else LI_ERR_SHAPE, nothing launched).
 * Accumulation is fp32 on the tensor cores; the softmax weights enter the P.V
 * product rounded to dtype.  Needs no workspace.  One launch (a thread-block
 * cluster per row when rows are few).
 */
#define LI_DEV_BAD_INDEX     0x20  /* sparse attention: an index outside [-1, Sk) (skipped) */
typedef struct {
    int32_t layout_q, layout_kv;
    int32_t dtype;
    int32_t B, S1, S2, T1, T2;
    int32_t N1, D, Dv;
    int32_t num_blocks, block_size, max_blocks_per_seq;
    int32_t sparse_count;
    float softmax_scale;
    int32_t reserved;
} li_sfa_params;

LI_API li_status li_sparse_attention(const li_sfa_params *p, const void *query, const void *key,
                                     const void *value, const int32_t *sparse_indices,
                                     const int32_t *act_seq_q, const int32_t *act_seq_k,
                                     const int32_t *block_table, void *out, float *lse,
                                     int32_t *status, void *stream);

/* Thread-local message describing the last non-OK status. */
LI_API const char *li_last_error(void);

/*
 * SYNCHRONISING: copy the device status word of `workspace` to the host after
 * everything queued on `stream` has finished.  *flags receives the LI_DEV_*
 * bits of the last call that used this workspace.  Returns LI_ERR_DEVICE when
 * any bit is set, LI_OK otherwise.
 */
LI_API li_status li_read_device_status(const void *workspace, void *stream, int32_t *flags);

/*
 * Self-test of the bounded wait used by every pipeline barrier: one thread
 * waits on a shared-memory barrier that nothing will ever complete, gives up
 * after timeout_ns nanoseconds and ORs LI_DEV_TIMEOUT into *status_word (a
 * device int32).  Lets a test check that an expired wait reports an error and
 * leaves the context usable, without faulting or hanging the GPU.
 */
LI_API li_status li_selftest_bounded_wait(int32_t *status_word, int64_t timeout_ns, void *stream);

/*
 * Per-stage timing: when `events` holds n >= 4 cudaEvent_t handles (passed as
 * void*), every later li_indexer / li_quant_indexer call on this thread records
 * events[0] before the scheduler, events[1] after it, events[2] after the score
 * kernel and events[3] after the Top-k kernel, on the call's stream.  n = 0 or
 * events = NULL turns it off.  The handles are borrowed, not owned.
 */
LI_API void li_set_profile_events(void *const *events, int32_t n);

/* Number of kernels launched by the last successful call on this thread. */
LI_API int32_t li_last_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* LI_H */
