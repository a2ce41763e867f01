// li_api.cu -- the C ABI of libli: argument checks, workspace layout, TMA
// descriptors and the three launches of one indexer call (scheduler, score,
// Top-k), all asynchronous on the caller's stream.
//
// The checks follow the constraints printed by the pages: the CANN guide's
// "约束说明" and "参数校验规则详解" (empty tensors rejected, layout matching,
// PA block size, q/k dtype equality, topk range, NaN undefined), the
// mindspore page's argument list (N2 = 1, D = 128, reserved pre/next tokens,
// TND needs actual_seq_lengths_query) and the README's "约束说明" (prefix
// sums for TND, PA needs actual_seq_lengths_key and a 2-D block_table).
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <utility>

#include "li_internal.cuh"
#include "ptx.cuh"

using namespace li;

namespace {

thread_local std::string g_error;
thread_local int32_t g_launches = 0;
thread_local cudaEvent_t g_prof[4] = {nullptr, nullptr, nullptr, nullptr};
thread_local bool g_prof_on = false;

bool prof_mark(int i, cudaStream_t s)
{
    return !g_prof_on || cudaEventRecord(g_prof[i], s) == cudaSuccess;
}

li_status fail(li_status s, const char *fmt, ...)
{
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_error = buf;
    return s;
}

constexpr int64_t kInt64Max = 0x7FFFFFFFFFFFFFFFLL;
constexpr int64_t kInt32Max = 0x7FFFFFFF;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

int elem_bytes(int dt) { return dt == LI_FP32 ? 4 : (dt == LI_FP8_E4M3 || dt == LI_INT8) ? 1 : 2; }

// Score-row capacity: the longest key sequence any batch may have.
int64_t key_bound(const li_params &p)
{
    if (p.max_seqlen_k > 0) return p.max_seqlen_k;
    if (p.layout_k == LI_BSND) return p.S2;
    if (p.layout_k == LI_TND) return p.T2;
    return (int64_t)p.max_blocks_per_seq * p.block_size;
}

int64_t query_rows(const li_params &p) { return p.layout_q == LI_BSND ? (int64_t)p.B * p.S1 : p.T1; }

li_status check_params(const li_params *pp, bool quant)
{
    if (!pp) return fail(LI_ERR_NULL, "params is NULL");
    const li_params &p = *pp;
    if (p.layout_q != LI_BSND && p.layout_q != LI_TND)
        return fail(LI_ERR_LAYOUT, "layout_q must be BSND or TND");
    if (p.layout_k != LI_BSND && p.layout_k != LI_TND && p.layout_k != LI_PA_BSND)
        return fail(LI_ERR_LAYOUT, "layout_k must be BSND, TND or PA_BSND");
    if (p.layout_k != LI_PA_BSND && p.layout_k != p.layout_q)
        return fail(LI_ERR_LAYOUT, "without paged keys layout_k must equal layout_q");
    if (p.B < 1) return fail(LI_ERR_SHAPE, "B must be >= 1 (empty tensors are rejected)");
    if (p.layout_q == LI_BSND && p.S1 < 1) return fail(LI_ERR_SHAPE, "S1 must be >= 1");
    if (p.layout_q == LI_TND && p.T1 < 1) return fail(LI_ERR_SHAPE, "T1 must be >= 1");
    if (p.layout_k == LI_BSND && p.S2 < 1) return fail(LI_ERR_SHAPE, "S2 must be >= 1");
    if (p.layout_k == LI_TND && p.T2 < 1) return fail(LI_ERR_SHAPE, "T2 must be >= 1");
    if (p.N2 != 1) return fail(LI_ERR_SHAPE, "N2 (key heads) must be 1");
    if (p.N1 < 1 || p.N1 > 64) return fail(LI_ERR_SHAPE, "N1 must be in [1, 64]");
    if (p.sparse_count < 1 || p.sparse_count > 8192)
        return fail(LI_ERR_SHAPE, "sparse_count must be in [1, 8192]");
    if (p.sparse_mode != 0 && p.sparse_mode != 3)
        return fail(LI_ERR_SHAPE, "sparse_mode must be 0 or 3");
    if (p.pre_tokens != kInt64Max || p.next_tokens != kInt64Max)
        return fail(LI_ERR_SHAPE, "pre_tokens/next_tokens only support their default 2^63-1");
    if (p.return_value != 0 && p.return_value != 1)
        return fail(LI_ERR_SHAPE, "return_value must be 0 or 1");
    if (p.max_seqlen_k < 0) return fail(LI_ERR_SHAPE, "max_seqlen_k must be >= 0");
    if (p.init_num < 0 || p.local_num < 0)
        return fail(LI_ERR_SHAPE, "init_num and local_num must be >= 0");
    if ((int64_t)p.init_num + p.local_num > p.sparse_count)
        return fail(LI_ERR_SHAPE, "init_num + local_num must not exceed sparse_count");
    if (p.cmp_ratio < 0 || p.cmp_ratio > 128 || (p.cmp_ratio & (p.cmp_ratio - 1)))
        return fail(LI_ERR_SHAPE, "cmp_ratio must be 0, 1 or a power of two up to 128");
    if (p.reserved != 0) return fail(LI_ERR_SHAPE, "reserved must be 0");
    if (quant) {
        if (p.dtype_qk != LI_FP8_E4M3 && p.dtype_qk != LI_INT8)
            return fail(LI_ERR_DTYPE, "li_quant_indexer takes fp8 e4m3 or int8 query/key");
        if (p.dtype_scale != LI_FP32 && p.dtype_scale != LI_FP16)
            return fail(LI_ERR_DTYPE, "dequant scales must be fp32 or fp16");
        if (p.D != 128) return fail(LI_ERR_SHAPE, "D must be 128 for 8-bit query/key");
    } else {
        if (p.dtype_qk != LI_BF16 && p.dtype_qk != LI_FP16)
            return fail(LI_ERR_DTYPE, "li_indexer takes bf16 or fp16 query/key");
        if (p.D != 128 && p.D != 64) return fail(LI_ERR_SHAPE, "D must be 128 (or 64)");
    }
    if (p.dtype_w != LI_BF16 && p.dtype_w != LI_FP16 && p.dtype_w != LI_FP32)
        return fail(LI_ERR_DTYPE, "weights must be bf16, fp16 or fp32");
    if (p.layout_k == LI_PA_BSND) {
        if (p.block_size < 16 || p.block_size > 1024 || p.block_size % 16)
            return fail(LI_ERR_SHAPE, "block_size must be a multiple of 16 in [16, 1024]");
        if (p.num_blocks < 1 || p.max_blocks_per_seq < 1)
            return fail(LI_ERR_SHAPE, "num_blocks and max_blocks_per_seq must be >= 1");
        const int64_t dense = (int64_t)p.block_size * p.N2 * p.D;
        if (p.key_block_stride != 0 && p.key_block_stride < dense)
            return fail(LI_ERR_SHAPE, "key_block_stride is smaller than one block");
        const int64_t stride = p.key_block_stride ? p.key_block_stride : dense;
        if ((stride * elem_bytes(p.dtype_qk)) % 16)
            return fail(LI_ERR_SHAPE, "key_block_stride must be a multiple of 16 bytes");
        if ((int64_t)p.max_blocks_per_seq * p.block_size > kInt32Max)
            return fail(LI_ERR_SHAPE, "paged key capacity exceeds int32");
    }
    const int64_t rows = query_rows(p);
    if (rows * p.N1 > kInt32Max) return fail(LI_ERR_SHAPE, "query rows x heads exceed int32");
    if (p.layout_k == LI_BSND && (int64_t)p.B * p.S2 > kInt32Max)
        return fail(LI_ERR_SHAPE, "key rows exceed int32");
    if (key_bound(p) > kInt32Max) return fail(LI_ERR_SHAPE, "max_seqlen_k exceeds int32");
    return LI_OK;
}

Tiling make_tiling(const li_params &p)
{
    Tiling t{};
    int n1p = 8;
    while (n1p < p.N1) n1p <<= 1;
    t.n1p = n1p;
    t.nq = 256 / n1p;
    t.chunks = p.D * elem_bytes(p.dtype_qk) / 128;
    t.stages = score_stages(t.chunks);
    t.smem = score_smem_bytes(t.chunks);
    return t;
}

WorkspaceLayout make_layout(const li_params &p, const Tiling &t)
{
    WorkspaceLayout w{};
    w.rows = query_rows(p);
    w.ld = (int64_t)align_up((size_t)key_bound(p), 4);
    w.max_blocks = (int32_t)(p.layout_q == LI_BSND ? (int64_t)p.B * ceil_div(p.S1, t.nq)
                                                    : ceil_div(p.T1, t.nq) + p.B);
    size_t off = 0;
    w.header = off;
    off += align_up(sizeof(PlanHeader), kAlign);
    w.batches = off;
    off += align_up(sizeof(BatchInfo) * (size_t)p.B, kAlign);
    w.blocks = off;
    off += align_up(sizeof(BlockInfo) * (size_t)w.max_blocks, kAlign);
    w.starts = off;
    off += align_up(sizeof(int4) * (size_t)kMaxScoreGrid, kAlign);
    w.scores = off;
    off += align_up(sizeof(float) * (size_t)w.rows * (size_t)w.ld, kAlign);
    w.total = off;
    return w;
}

// ---- TMA descriptor encoding through the driver entry point (no -lcuda)
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

li_status encode(CUtensorMap *m, int es, const void *base, int rank, const uint64_t *dims,
                 const uint64_t *strides_bytes, const uint32_t *box, const char *what)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(LI_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    cuuint64_t d[4], s[3];
    cuuint32_t b[4], e[4] = {1, 1, 1, 1};
    for (int i = 0; i < rank; ++i) { d[i] = dims[i]; b[i] = box[i]; }
    for (int i = 0; i + 1 < rank; ++i) s[i] = strides_bytes[i];
    CUresult r = fn(m, es == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16,
                    (cuuint32_t)rank, const_cast<void *>(base), d, s, b, e,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(LI_ERR_CUDA, "tensor map for %s rejected (CUresult %d)", what, (int)r);
    return LI_OK;
}

int num_sms()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return n;
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int topk_cap(int64_t ld, int k, int kmax)
{
    // rows of up to 16384 keys are cached in shared memory (at most ~100 KB
    // per CTA, two CTAs per SM); longer rows stream from L2
    int64_t cap = 16384;
    if (cap > ld) cap = ld;
    (void)k;
    (void)kmax;
    return (int)((cap + 3) & ~int64_t(3));
}

li_status run(const li_params *pp, bool quant, const void *query, const void *key,
              const void *weights, const void *q_scale, const void *k_scale,
              const int32_t *act_q, const int32_t *act_k, const int32_t *block_table,
              int32_t *out_idx, float *out_val, void *workspace, size_t ws_bytes, void *stream)
{
    g_launches = 0;
    li_status st = check_params(pp, quant);
    if (st != LI_OK) return st;
    const li_params &p = *pp;
    if (!query || !key || !weights || !out_idx)
        return fail(LI_ERR_NULL, "query, key, weights and sparse_indices are required");
    if (p.return_value && !out_val) return fail(LI_ERR_NULL, "return_value=1 needs sparse_values");
    if (!p.return_value && out_val)
        return fail(LI_ERR_NULL, "sparse_values must be NULL when return_value=0");
    if (quant && (!q_scale || !k_scale)) return fail(LI_ERR_NULL, "dequant scales are required");
    if (p.layout_q == LI_TND && !act_q)
        return fail(LI_ERR_NULL, "TND query needs actual_seq_lengths_query (prefix sums)");
    if ((p.layout_k == LI_TND || p.layout_k == LI_PA_BSND) && !act_k)
        return fail(LI_ERR_NULL, "TND/PA key needs actual_seq_lengths_key");
    if (p.layout_k == LI_PA_BSND && !block_table) return fail(LI_ERR_NULL, "PA needs block_table");
    int cmp_shift = 0;
    while ((1 << cmp_shift) < p.cmp_ratio) ++cmp_shift;
    if (cmp_shift > 0 && p.sparse_mode == 3 && !p.cmp_residual_k)
        return fail(LI_ERR_NULL, "cmp_ratio > 1 with sparse_mode 3 needs cmp_residual_k");
    if (!aligned(query, 16) || !aligned(key, 16))
        return fail(LI_ERR_SHAPE, "query and key must be 16-byte aligned");
    if (!aligned(weights, 4) || !aligned(out_idx, 4) || (out_val && !aligned(out_val, 4)))
        return fail(LI_ERR_SHAPE, "weights and outputs must be 4-byte aligned");
    if (quant && (!aligned(q_scale, p.dtype_scale == LI_FP32 ? 4 : 2) ||
                  !aligned(k_scale, p.dtype_scale == LI_FP32 ? 4 : 2)))
        return fail(LI_ERR_SHAPE, "dequant scales must be aligned to their element size");
    const Tiling t = make_tiling(p);
    const WorkspaceLayout w = make_layout(p, t);
    if (!workspace) return fail(LI_ERR_WORKSPACE, "workspace is NULL");
    if (!aligned(workspace, kAlign)) return fail(LI_ERR_WORKSPACE, "workspace must be 256-byte aligned");
    if (ws_bytes < w.total)
        return fail(LI_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", ws_bytes, w.total);
    const int sms = num_sms();
    if (sms <= 0) return fail(LI_ERR_CUDA, "no CUDA device");
    if (sms > kMaxScoreGrid) return fail(LI_ERR_CUDA, "more than %d SMs", kMaxScoreGrid);

    const int es = elem_bytes(p.dtype_qk);
    const int inner = 128 / es;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    PlanHeader *hdr = reinterpret_cast<PlanHeader *>(ws + w.header);
    BatchInfo *batches = reinterpret_cast<BatchInfo *>(ws + w.batches);
    BlockInfo *blocks = reinterpret_cast<BlockInfo *>(ws + w.blocks);
    float *scores = reinterpret_cast<float *>(ws + w.scores);

    // Tensor maps.  With 256-byte operand rows (bf16/fp16, D = 128) a row is
    // two 128-byte swizzle chunks; an outer map dimension of extent 2 and
    // stride 128 B walks them, so one copy fills both chunk planes of a tile
    // ([chunk][row][128 B] in shared memory).  Otherwise one copy per chunk.
    CUtensorMap qmap, kmap;
    const int q_box_rows = (p.N1 == t.n1p) ? 256 : p.N1;
    const bool two = t.chunks == 2;
    int q_single = 0, k_single = 0;
    if (two && q_box_rows == 256) {
        const uint64_t dims[3] = {(uint64_t)inner, (uint64_t)(w.rows * p.N1), 2};
        const uint64_t strides[2] = {(uint64_t)p.D * es, 128};
        const uint32_t box[3] = {(uint32_t)inner, 256, 2};
        if ((st = encode(&qmap, es, query, 3, dims, strides, box, "query")) != LI_OK) return st;
        q_single = 1;
    } else {
        const uint64_t dims[2] = {(uint64_t)p.D, (uint64_t)(w.rows * p.N1)};
        const uint64_t strides[1] = {(uint64_t)p.D * es};
        const uint32_t box[2] = {(uint32_t)inner, (uint32_t)q_box_rows};
        if ((st = encode(&qmap, es, query, 2, dims, strides, box, "query")) != LI_OK) return st;
    }
    int pa_box_rows = 0;
    if (p.layout_k != LI_PA_BSND) {
        const int64_t krows = p.layout_k == LI_BSND ? (int64_t)p.B * p.S2 : p.T2;
        if (two) {
            const uint64_t dims[3] = {(uint64_t)inner, (uint64_t)krows, 2};
            const uint64_t strides[2] = {(uint64_t)p.D * es, 128};
            const uint32_t box[3] = {(uint32_t)inner, (uint32_t)kTileKeys, 2};
            if ((st = encode(&kmap, es, key, 3, dims, strides, box, "key")) != LI_OK) return st;
            k_single = 1;
        } else {
            const uint64_t dims[2] = {(uint64_t)p.D, (uint64_t)krows};
            const uint64_t strides[1] = {(uint64_t)p.D * es};
            const uint32_t box[2] = {(uint32_t)inner, (uint32_t)kTileKeys};
            if ((st = encode(&kmap, es, key, 2, dims, strides, box, "key")) != LI_OK) return st;
        }
    } else {
        int g = 128;
        while (p.block_size % g) g >>= 1;               // gcd(block_size, 128) >= 16
        pa_box_rows = g;
        const int64_t stride = p.key_block_stride ? p.key_block_stride
                                                  : (int64_t)p.block_size * p.N2 * p.D;
        if (two && g == kTileKeys) {
            const uint64_t dims[4] = {(uint64_t)inner, (uint64_t)p.block_size, 2, (uint64_t)p.num_blocks};
            const uint64_t strides[3] = {(uint64_t)p.D * p.N2 * es, 128, (uint64_t)stride * es};
            const uint32_t box[4] = {(uint32_t)inner, (uint32_t)g, 2, 1};
            if ((st = encode(&kmap, es, key, 4, dims, strides, box, "paged key")) != LI_OK) return st;
            k_single = 1;
        } else {
            const uint64_t dims[3] = {(uint64_t)p.D, (uint64_t)p.block_size, (uint64_t)p.num_blocks};
            const uint64_t strides[2] = {(uint64_t)p.D * p.N2 * es, (uint64_t)stride * es};
            const uint32_t box[3] = {(uint32_t)inner, (uint32_t)g, 1};
            if ((st = encode(&kmap, es, key, 3, dims, strides, box, "paged key")) != LI_OK) return st;
        }
    }

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    PlanArgs pa{};
    pa.act_q = act_q;
    pa.act_k = act_k;
    pa.batches = batches;
    pa.blocks = blocks;
    pa.hdr = hdr;
    pa.layout_q = p.layout_q;
    pa.layout_k = p.layout_k;
    pa.mode = p.sparse_mode;
    pa.B = p.B;
    pa.S1 = p.S1;
    pa.S2 = p.S2;
    pa.T1 = p.T1;
    pa.T2 = p.T2;
    pa.nq = t.nq;
    pa.cta_start = reinterpret_cast<int4 *>(ws + w.starts);
    pa.grid = sms;
    pa.max_blocks = w.max_blocks;
    pa.ld = w.ld;
    pa.pa_capacity = (int64_t)p.max_blocks_per_seq * p.block_size;
    pa.cmp_res = cmp_shift > 0 && p.sparse_mode == 3 ? p.cmp_residual_k : nullptr;
    pa.cmp_shift = cmp_shift;
    pa.q_cost = quant ? kQCost8 : kQCost16;
    if (!prof_mark(0, s)) return fail(LI_ERR_CUDA, "recording profile event 0 failed");
    cudaError_t e = launch_plan(pa, s);
    if (e != cudaSuccess) return fail(LI_ERR_CUDA, "scheduler launch: %s", cudaGetErrorString(e));
    ++g_launches;
    if (!prof_mark(1, s)) return fail(LI_ERR_CUDA, "recording profile event 1 failed");

    ScoreArgs sa{};
    sa.weights = weights;
    sa.q_scale = q_scale;
    sa.k_scale = k_scale;
    sa.block_table = block_table;
    sa.batches = batches;
    sa.blocks = blocks;
    sa.cta_start = reinterpret_cast<const int4 *>(ws + w.starts);
    sa.hdr = hdr;
    sa.scores = scores;
    sa.ld = w.ld;
    sa.N1 = p.N1;
    sa.mode = p.sparse_mode;
    sa.is_pa = p.layout_k == LI_PA_BSND;
    sa.quant = quant ? 1 : 0;
    sa.dtype_w = p.dtype_w;
    sa.block_size = p.block_size;
    sa.max_blocks_per_seq = p.max_blocks_per_seq;
    sa.num_blocks = p.num_blocks;
    sa.pa_box_rows = pa_box_rows;
    sa.q_box_rows = q_box_rows;
    sa.q_single = q_single;
    sa.k_single = k_single;
    // operand formats: f16 0 / bf16 1 (kind::f16), e4m3 0 (kind::f8f6f4),
    // signed 8-bit 1 with an s32 accumulator (kind::i8)
    const int kind = !quant ? kKindF16 : (p.dtype_qk == LI_INT8 ? kKindI8 : kKindE4M3);
    const uint32_t fmt = kind == kKindF16 ? (p.dtype_qk == LI_BF16 ? 1u : 0u) : (kind == kKindI8 ? 1u : 0u);
    sa.idesc_base = make_idesc(fmt, fmt, 128, 0, kind == kKindI8 ? 2u : 1u);
    sa.cmp_shift = cmp_shift;
    sa.q_cost = pa.q_cost;
    sa.dtype_scale = p.dtype_scale;
    sa.timeout_ns = kDefaultTimeoutNs;
    e = launch_score(sa, t, qmap, kmap, kind, sms, s);
    if (e != cudaSuccess) return fail(LI_ERR_CUDA, "score launch: %s", cudaGetErrorString(e));
    ++g_launches;
    if (!prof_mark(2, s)) return fail(LI_ERR_CUDA, "recording profile event 2 failed");

    TopkArgs ta{};
    ta.scores = scores;
    ta.ld = w.ld;
    ta.row_len = nullptr;
    ta.batches = batches;
    ta.B = p.B;
    ta.layout_q = p.layout_q;
    ta.S1 = p.S1;
    ta.mode = p.sparse_mode;
    ta.rows = (int32_t)w.rows;
    ta.k = p.sparse_count;
    ta.out_idx = out_idx;
    ta.out_val = out_val;
    ta.kmax = (p.sparse_count + 31) & ~31;
    ta.cap = topk_cap(w.ld, p.sparse_count, ta.kmax);
    ta.standalone = 0;
    ta.init_num = p.init_num;
    ta.local_num = p.local_num;
    ta.cmp_shift = cmp_shift;
    e = launch_topk(ta, s);
    if (e != cudaSuccess) return fail(LI_ERR_CUDA, "top-k launch: %s", cudaGetErrorString(e));
    ++g_launches;
    if (!prof_mark(3, s)) return fail(LI_ERR_CUDA, "recording profile event 3 failed");
    return LI_OK;
}

}  // namespace

namespace li {

uint64_t current_context_id()
{
    typedef CUresult (*GetCurrentFn)(CUcontext *);
    typedef CUresult (*GetIdFn)(CUcontext, unsigned long long *);
    static GetCurrentFn get_current = nullptr;
    static GetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<GetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<GetIdFn>(p);
    });
    if (!get_current || !get_id) return 0;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
    unsigned long long id = 0;
    if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

cudaError_t set_max_dynamic_smem(const void *kern, int bytes)
{
    static std::mutex mu;
    static std::map<std::pair<const void *, uint64_t>, int> done;
    const uint64_t ctx = current_context_id();
    if (ctx) {
        std::lock_guard<std::mutex> lock(mu);
        auto it = done.find({kern, ctx});
        if (it != done.end() && it->second >= bytes) return cudaSuccess;
    }
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    const uint64_t ctx_after = current_context_id();   // the call may have made the context current
    if (ctx_after) {
        std::lock_guard<std::mutex> lock(mu);
        int &v = done[{kern, ctx_after}];
        if (v < bytes) v = bytes;
    }
    return cudaSuccess;
}

// Record `msg` as the thread's last error and return `s` (for the other
// translation units of the library).
li_status report_error(li_status s, const char *msg) { return fail(s, "%s", msg); }
void set_launch_count(int32_t n) { g_launches = n; }
}  // namespace li

extern "C" {

li_status li_output_shape(const li_params *p, int64_t out_dims[4], int32_t *ndim)
{
    if (!out_dims || !ndim) return fail(LI_ERR_NULL, "out_dims and ndim are required");
    li_status st = check_params(p, p && (p->dtype_qk == LI_FP8_E4M3 || p->dtype_qk == LI_INT8));
    if (st != LI_OK) return st;
    if (p->layout_q == LI_BSND) {
        out_dims[0] = p->B;
        out_dims[1] = p->S1;
        out_dims[2] = p->N2;
        out_dims[3] = p->sparse_count;
        *ndim = 4;
    } else {
        out_dims[0] = p->T1;
        out_dims[1] = p->N2;
        out_dims[2] = p->sparse_count;
        out_dims[3] = 0;
        *ndim = 3;
    }
    return LI_OK;
}

li_status li_workspace_size(const li_params *p, size_t *bytes)
{
    if (!bytes) return fail(LI_ERR_NULL, "bytes is NULL");
    li_status st = check_params(p, p && (p->dtype_qk == LI_FP8_E4M3 || p->dtype_qk == LI_INT8));
    if (st != LI_OK) return st;
    *bytes = make_layout(*p, make_tiling(*p)).total;
    return LI_OK;
}

li_status li_indexer(const li_params *p, const void *query, const void *key, const void *weights,
                     const int32_t *act_seq_q, const int32_t *act_seq_k,
                     const int32_t *block_table, int32_t *sparse_indices, float *sparse_values,
                     void *workspace, size_t workspace_bytes, void *stream)
{
    return run(p, false, query, key, weights, nullptr, nullptr, act_seq_q, act_seq_k, block_table,
               sparse_indices, sparse_values, workspace, workspace_bytes, stream);
}

li_status li_quant_indexer(const li_params *p, const void *query, const void *key,
                           const void *weights, const void *q_scale, const void *k_scale,
                           const int32_t *act_seq_q, const int32_t *act_seq_k,
                           const int32_t *block_table, int32_t *sparse_indices,
                           float *sparse_values, void *workspace, size_t workspace_bytes,
                           void *stream)
{
    return run(p, true, query, key, weights, q_scale, k_scale, act_seq_q, act_seq_k, block_table,
               sparse_indices, sparse_values, workspace, workspace_bytes, stream);
}

li_status li_topk(const float *scores, int64_t ld, const int32_t *row_len, int32_t rows,
                  int32_t k, int32_t *sparse_indices, float *sparse_values, void *stream)
{
    g_launches = 0;
    if (!scores || !sparse_indices) return fail(LI_ERR_NULL, "scores and sparse_indices are required");
    if (rows < 0) return fail(LI_ERR_SHAPE, "rows must be >= 0");
    if (k < 1 || k > 8192) return fail(LI_ERR_SHAPE, "k must be in [1, 8192]");
    if (ld < 1 || ld % 4 || ld > kInt32Max) return fail(LI_ERR_SHAPE, "ld must be a positive multiple of 4");
    if (!aligned(scores, 16)) return fail(LI_ERR_SHAPE, "scores must be 16-byte aligned");
    TopkArgs ta{};
    ta.scores = scores;
    ta.ld = ld;
    ta.row_len = row_len;
    ta.rows = rows;
    ta.k = k;
    ta.out_idx = sparse_indices;
    ta.out_val = sparse_values;
    ta.kmax = (k + 31) & ~31;
    ta.cap = topk_cap(ld, k, ta.kmax);
    ta.standalone = 1;
    cudaError_t e = launch_topk(ta, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(LI_ERR_CUDA, "top-k launch: %s", cudaGetErrorString(e));
    g_launches = rows > 0 ? 1 : 0;
    return LI_OK;
}

const char *li_last_error(void) { return g_error.c_str(); }

li_status li_read_device_status(const void *workspace, void *stream, int32_t *flags)
{
    if (!workspace || !flags) return fail(LI_ERR_NULL, "workspace and flags are required");
    int32_t v = 0;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(&v, workspace, sizeof v, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return fail(LI_ERR_CUDA, "reading the status word: %s", cudaGetErrorString(e));
    *flags = v;
    if (v) return fail(LI_ERR_DEVICE, "device status 0x%x", v);
    return LI_OK;
}

li_status li_selftest_bounded_wait(int32_t *status_word, int64_t timeout_ns, void *stream)
{
    if (!status_word) return fail(LI_ERR_NULL, "status_word is NULL");
    if (timeout_ns < 0) return fail(LI_ERR_SHAPE, "timeout_ns must be >= 0");
    cudaError_t e = launch_wait_selftest(status_word, timeout_ns, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(LI_ERR_CUDA, "self-test launch: %s", cudaGetErrorString(e));
    g_launches = 1;
    return LI_OK;
}

void li_set_profile_events(void *const *events, int32_t n)
{
    g_prof_on = events != nullptr && n >= 4;
    for (int i = 0; i < 4; ++i) g_prof[i] = g_prof_on ? static_cast<cudaEvent_t>(events[i]) : nullptr;
}

int32_t li_last_launch_count(void) { return g_launches; }

}  // extern "C"
