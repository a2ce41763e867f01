// li_internal.cuh -- structures shared by the host API and the kernels of
// libli: the workspace layout written by the scheduler and the launch
// arguments of the score and Top-k kernels.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/li.h"

namespace li {

constexpr int kTileKeys = 128;        // keys per MMA tile (the M axis)
constexpr int kAccCols = 256;         // TMEM columns per accumulator (the N axis)
constexpr int kAccStages = 2;         // double-buffered accumulators (512 TMEM columns)
constexpr int kGroupWarps = 8;        // warps of one epilogue group (2 per TMEM lane quarter)
constexpr int kEpiWarps = kAccStages * kGroupWarps;   // one group per accumulator
// Scheduler weight of one query-tile load, in key tiles: the bubble a block
// switch costs relative to one tile's work.  8-bit keys make a tile cheaper
// (half the MMA time and bytes), so a block switch weighs more.
constexpr int kQCost16 = 2;           // bf16 / fp16 q/k
constexpr int kQCost8 = 4;            // fp8 / int8 q/k
constexpr int kScoreThreads = 32 * (2 + kEpiWarps);
constexpr int kTopkThreads = 512;
constexpr int kPlanThreads = 1024;
constexpr size_t kAlign = 256;
constexpr int kMaxScoreGrid = 1024;   // score CTAs whose start the scheduler records
constexpr int64_t kDefaultTimeoutNs = 2000000000LL;   // 2 s per pipeline wait

// Per-batch sequence bookkeeping, clamped to what the tensors can hold.
struct BatchInfo {
    int32_t q_off;     // token row of query/weights for i = 0
    int32_t Sq;        // query length
    int32_t k_off;     // key row for t = 0 (BSND/TND; 0 for PA)
    int32_t Sk;        // key length
    int32_t blk_off;   // first query block of this batch
    int32_t row0;      // output row of i = 0
    int32_t nblk;      // query blocks of this batch
    int32_t res;       // residual original key tokens (compressed keys, mode 3)
};

// Keys visible to query i under right-down causal masking (CANN
// LightningIndexerV2 guide, sparse_mode 3, with cmp_ratio = 2^shift): each
// key stands for 2^shift original tokens, the batch has Sk * 2^shift + res
// original key tokens, and a key is visible once its last original token is
// at or before position i + that length - Sq.  shift = res = 0: t <= i + Sk - Sq.
__host__ __device__ __forceinline__ int32_t causal_visible(int64_t i, int32_t Sq, int32_t Sk,
                                                           int32_t res, int32_t shift)
{
    const int64_t v = (i + 1 - Sq + ((int64_t)Sk << shift) + res) >> shift;   // floor
    return v < 0 ? 0 : (v > Sk ? Sk : (int32_t)v);
}

// One query block: up to nq consecutive queries of one batch.
struct BlockInfo {
    int32_t b;
    int32_t i0;          // first query position
    int32_t unit_start;  // first work unit (key tile) of this block
    int32_t ntiles;      // visible key tiles of the block's last query
};

// Head of the workspace (256 bytes): the device status word and plan totals.
struct PlanHeader {
    int32_t status;        // LI_DEV_* bits
    int32_t total_blocks;
    int32_t total_units;
    int32_t pad[61];
};

// Workspace carve-up (all offsets 256-byte aligned).
struct WorkspaceLayout {
    size_t header, batches, blocks, starts, scores, total;
    int64_t ld;           // floats per score row
    int64_t rows;         // query rows
    int32_t max_blocks;   // capacity of the block table
};

// Tiling chosen on the host for one call.
struct Tiling {
    int n1p;       // heads padded to a power of two >= 8
    int nq;        // queries per block = 256 / n1p
    int chunks;    // 128-byte column chunks per operand row (D * elem bytes / 128)
    int stages;    // key-tile pipeline depth
    size_t smem;   // dynamic shared memory of the score kernel
};

struct PlanArgs {
    const int32_t *act_q, *act_k;
    BatchInfo *batches;
    BlockInfo *blocks;
    PlanHeader *hdr;
    int32_t layout_q, layout_k, mode;
    int32_t B, S1, S2, T1, T2;
    int32_t nq, max_blocks;
    int64_t ld;            // score row capacity: key lengths are clamped to it
    int64_t pa_capacity;   // max_blocks_per_seq * block_size
    int4 *cta_start;       // per score CTA: (block, tile, block's unit_start, block's ntiles)
    int32_t grid;          // score CTAs
    const int32_t *cmp_res;  // [B] residual original key tokens (NULL: none)
    int32_t cmp_shift;       // log2(cmp_ratio)
    int32_t q_cost;          // weight of a query-tile load (kQCost16 or kQCost8)
};

struct ScoreArgs {
    const void *weights;
    const void *q_scale;        // dequant scales, dtype_scale (fp32 or fp16)
    const void *k_scale;
    const int32_t *block_table;
    const BatchInfo *batches;
    const BlockInfo *blocks;
    const int4 *cta_start;      // where each CTA's share of the work list begins
    PlanHeader *hdr;
    float *scores;
    int64_t ld;
    int32_t N1, mode, is_pa, quant;
    int32_t dtype_w, dtype_scale;
    int32_t block_size, max_blocks_per_seq, num_blocks, pa_box_rows;
    int32_t q_box_rows;         // rows per Q TMA box: n1p*nq (packed) or N1 (per query)
    int32_t q_single, k_single; // one copy covers both 128-byte chunks (3-D / 4-D maps)
    uint32_t idesc_base;        // instruction descriptor without N
    int32_t cmp_shift;          // log2(cmp_ratio): compressed keys under mode 3
    int32_t q_cost;             // weight of a query-tile load in the work list
    int64_t timeout_ns;
};

struct TopkArgs {
    const float *scores;
    int64_t ld;
    const int32_t *row_len;          // standalone mode: per-row candidate count (or NULL)
    const BatchInfo *batches;        // indexer mode: per-batch info (row_len == NULL)
    int32_t B, layout_q, S1, mode;
    int32_t rows, k;
    int32_t *out_idx;
    float *out_val;
    int32_t cap;                     // row elements cached in shared memory
    int32_t kmax;                    // capacity of the selection buffers (>= k)
    int32_t standalone;
    int32_t init_num, local_num;     // always-selected sink keys and local window
    int32_t cmp_shift;               // log2(cmp_ratio): compressed keys under mode 3
};

size_t topk_smem_bytes(int cap, int kmax);
size_t score_smem_bytes(int chunks);
int score_stages(int chunks);

cudaError_t launch_plan(const PlanArgs &a, cudaStream_t s);
// Operand kinds of the score MMA.
enum ScoreKind { kKindF16 = 0, kKindE4M3 = 1, kKindI8 = 2 };
cudaError_t launch_score(const ScoreArgs &a, const Tiling &t, const CUtensorMap &qmap,
                         const CUtensorMap &kmap, int kind, int grid, cudaStream_t s);
cudaError_t launch_topk(const TopkArgs &a, cudaStream_t s);
cudaError_t launch_wait_selftest(int32_t *status, int64_t timeout_ns, cudaStream_t s);

// Unique id of the calling thread's current CUDA context (the driver's
// cuCtxGetId), or 0 when there is none or it cannot be read.  Ids are never
// reused within a process, so a context re-created after cudaDeviceReset
// gets a new one.
uint64_t current_context_id();
// Raise `kern`'s dynamic shared-memory limit to `bytes` once per kernel and
// context (cudaFuncSetAttribute on the first launch in a context only).
cudaError_t set_max_dynamic_smem(const void *kern, int bytes);

}  // namespace li
