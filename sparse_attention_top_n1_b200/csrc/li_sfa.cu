// li_sfa.cu -- sparse attention over the indexer's selected keys, on the
// 5th-generation tensor cores.
//
// The consumer of the indexer's output (CANN TileLang LightningIndexer guide,
// section "LightningIndexer 在稀疏注意力中的地位": the index tensor names, for
// every query token, the key/value subset its attention runs over).  For
// query row r of batch b and head h:
//
//     out_h = sum_{j in J} softmax_j(scale * q_h . k_j) * v_j,   J = valid entries
//     lse_h = log sum_{j in J} exp(scale * q_h . k_j)
//
// One CTA per query row (or, when rows are few, a cluster of up to 8 CTAs per
// row, each taking a share of its keys, merged through distributed shared
// memory), two CTAs per SM, warp-specialised; the row's selected keys are
// taken 64 at a time:
//   warps 0-1  resolve each slot to a key row (batch offset, or the block
//              table for a paged pool; an empty or invalid slot becomes a
//              masked zero row) and gather the 64 key rows and 64 value rows
//              with 16-byte cp.async copies, one 256-byte row per half warp
//              and instruction, into a two-stage key ring and a three-stage
//              value ring in the 128-byte-swizzled layout the tensor core
//              reads; each thread's arrival on a stage's full barrier is
//              deferred by the copy unit until its copies have landed; the
//              tile's slot-validity mask goes to a ring of its own;
//   warp 2     issues S = Q K^T on tcgen05.mma (M = the heads, 64 or 128
//              rows with zero rows for N1 < 64; N = 64 keys; K = D = 128)
//              into one of two tensor-memory buffers, one tile ahead of
//              O += P V (A = the weights, K-major; B = the value tile read
//              MN-major from its gathered layout; fp32 accumulation in
//              tensor memory);
//   warps 3-6  the softmax: each reads its quarter of S out of tensor memory
//              (M = 64: four threads per head with the 16-lane load shape,
//              combined by two shuffles; M = 128: one thread per head), scales
//              the logits into the log2 domain, masks empty slots, rounds the
//              weights exp2(s - m) to the input type and writes them to the
//              shared-memory weights tile once the previous P V has read it
//              (the normaliser sums the same rounded values, so the output
//              stays a convex combination of values); the running max m
//              moves only when a tile's max beats it by more than 2^8, and
//              only then is O rescaled in tensor memory, so the weights stay
//              below 256 and O is touched rarely.
// out = O / l and lse = ln 2 * (m + log2 l) are written once per row.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cooperative_groups.h>

#include <cmath>
#include <cstdio>
#include <cstdint>

#include "li.h"
#include "ptx.cuh"

namespace li {
li_status report_error(li_status s, const char *msg);
void set_launch_count(int32_t n);
cudaError_t set_max_dynamic_smem(const void *kern, int bytes);
}  // namespace li

namespace {

using namespace li;

constexpr int kHd = 128;                  // D = Dv
constexpr int kSlots = 64;                // selected keys per tile: the N of S, the K of P.V
constexpr int kThreads = 224;             // two producer warps, MMA issuer, four softmax warps
constexpr int kProducers = 64;            // one producer thread per slot of a tile
constexpr int kKStages = 2, kVStages = 3;
constexpr int kMaskRing = 8;             // slot-validity masks in flight (>= kKStages + 2)
constexpr int kStageBytes = kSlots * kHd * 2;   // one key or value tile: two 64-column planes
constexpr int kPlane = kSlots * 128;            // one 64-column plane of a tile
constexpr int kMaxSplit = 8;              // CTAs (one cluster) sharing a row's keys
constexpr float kRescaleLog2 = 8.f;       // the running max moves when a tile beats it by 2^8

struct SfaArgs {
    const uint16_t *q, *k, *v;
    const int32_t *idx;
    const int32_t *act_q, *act_k, *block_table;
    uint16_t *out;
    float *lse;
    int32_t *status;
    int32_t layout_q, layout_kv;
    int32_t B, S1, S2, T1, T2, N1, K;
    int32_t num_blocks, block_size, max_blocks_per_seq;
    float scale_log2;                     // softmax scale * log2(e)
    int32_t bs_shift;                     // log2(block_size), or -1
};

// Shared memory of one CTA (byte offsets from a 1024-byte aligned base).  Q,
// the key and value tiles and the weights are stored as 128-byte rows in
// 64-column planes, 16-byte chunk c of row r at chunk position c ^ (r & 7)
// (the 128-byte swizzle of TMA and of the tensor core's descriptors).
template <int M>
struct Layout {
    static constexpr int QPLANE = M * 128;                  // M rows x 64 columns of 16 bits
    static constexpr int Q = 0;                             // [2][M][128 B]
    static constexpr int K = Q + 2 * QPLANE;                // [kKStages][2][64][128 B]
    static constexpr int V = K + kKStages * kStageBytes;    // [kVStages][2][64][128 B]
    static constexpr int P = V + kVStages * kStageBytes;    // [M][128 B]: weights, 64 keys along K
    static constexpr int MASK = P + QPLANE;                 // uint32 [kMaskRing][2]
    static constexpr int BARS = MASK + kMaskRing * 8;       // mbarriers
    static constexpr int NBARS = 2 * kKStages + 2 * kVStages + 2 + 2 + 1 + 1 + kMaskRing;
    static constexpr int TSLOT = BARS + NBARS * 8;         // TMEM address, then the abort flag
    static constexpr int MERGE = TSLOT + 16;                // float [3][128]: a cluster's (m, l), merge weights
    static constexpr int END = MERGE + 3 * 128 * 4;
    static constexpr int BYTES = END + 1024;                // + alignment of the base
};

__device__ __forceinline__ int32_t clampi(int64_t v, int64_t lo, int64_t hi)
{
    return (int32_t)(v < lo ? lo : (v > hi ? hi : v));
}

// Offset of 16-byte chunk `ch` (0..15) of row `r` in a two-plane tile.
__device__ __forceinline__ uint32_t chunk_off(int r, int ch, int plane_bytes)
{
    return (uint32_t)((ch >> 3) * plane_bytes + r * 128 + (((ch & 7) ^ (r & 7)) << 4));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
                 : "memory");
}
// Arrive on `bar` once all earlier cp.async copies of this thread have landed;
// the arrival counts towards the barrier's expected count (no increment).
__device__ __forceinline__ void cp_async_arrive(uint64_t *bar)
{
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

template <bool F16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi)
{
    if constexpr (F16) {
        const __half2 h = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<const uint32_t *>(&h);
    } else {
        const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<const uint32_t *>(&h);
    }
}

template <bool F16>
__device__ __forceinline__ float unpack_lo(uint32_t v)
{
    if constexpr (F16) return __half2float(__ushort_as_half((unsigned short)(v & 0xFFFFu)));
    else return __uint_as_float(v << 16);
}

template <bool F16>
__device__ __forceinline__ float unpack_hi(uint32_t v)
{
    if constexpr (F16) return __half2float(__ushort_as_half((unsigned short)(v >> 16)));
    else return __uint_as_float(v & 0xFFFF0000u);
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Columns 16*CH .. 16*CH+15 of this warp's lanes into r[16*CH ..].
template <int CH, int N>
__device__ __forceinline__ void tmem_ld16_into(uint32_t taddr, uint32_t (&r)[N])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[16 * CH + 0]), "=r"(r[16 * CH + 1]), "=r"(r[16 * CH + 2]), "=r"(r[16 * CH + 3]),
          "=r"(r[16 * CH + 4]), "=r"(r[16 * CH + 5]), "=r"(r[16 * CH + 6]), "=r"(r[16 * CH + 7]),
          "=r"(r[16 * CH + 8]), "=r"(r[16 * CH + 9]), "=r"(r[16 * CH + 10]), "=r"(r[16 * CH + 11]),
          "=r"(r[16 * CH + 12]), "=r"(r[16 * CH + 13]), "=r"(r[16 * CH + 14]), "=r"(r[16 * CH + 15])
        : "r"(taddr + 16 * CH));
}

// 16 lanes x 256 bits, 8 repetitions (64 columns): thread t gets lanes
// t/4 and t/4 + 8, columns 8j + 2(t%4) and 8j + 2(t%4) + 1 in r[4j .. 4j+3]
// (lane t/4: r[4j], r[4j+1]; lane t/4 + 8: r[4j+2], r[4j+3]).
__device__ __forceinline__ void tmem_ld_16x256b_x8(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x8.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_st_16x256b_x8(uint32_t taddr, const uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.st.sync.aligned.16x256b.x8.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
        "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
        "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

// 2^x on the special-function unit (relative error about 2^-22, far below
// the 16-bit rounding the weights get next); 2^-inf = 0.
__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// max of three (one instruction on sm_100)
__device__ __forceinline__ float fmax3(float x, float y, float z)
{
    float m;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(m) : "f"(x), "f"(y), "f"(z));
    return m;
}

// (d0, d1) = (a0 * b0 + c0, a1 * b1 + c1) as one packed fp32 instruction
__device__ __forceinline__ void ffma2(float &d0, float &d1, float a0, float a1, float b0, float b1, float c0,
                                      float c1)
{
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d0), "=f"(d1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}

// (d0, d1) += (x0, x1) as one packed fp32 instruction
__device__ __forceinline__ void fadd2(float &d0, float &d1, float x0, float x1)
{
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%0, %1};\n\tmov.b64 rb, {%2, %3};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "+f"(d0), "+f"(d1)
        : "f"(x0), "f"(x1));
}

// Bounded wait on an mbarrier phase.  A wait that expires (2 s) flags
// LI_DEV_TIMEOUT and sets the CTA's abort flag; from then on every wait of
// the CTA returns after one suspended try (at most about a microsecond), and
// so does a wait of another CTA once it sees the flag in `status`, so a
// broken pipeline ends the kernel promptly (results are then undefined; the
// context stays usable).
__device__ __forceinline__ void wait_phase(uint64_t *bar, uint32_t parity, int32_t *status, volatile int *abort)
{
    // the waiting thread is suspended in hardware (up to 1 us per try) until
    // the phase completes, instead of spinning on the issue slots
    if (mbar_try_wait(bar, parity)) return;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1; !mbar_try_wait_sleep(bar, parity, 1000u); ++it) {
        if (*abort) return;
        // another CTA's timeout, looked at every 256 tries (a global load)
        if ((it & 255u) == 0 && status && (*reinterpret_cast<volatile int32_t *>(status) & LI_DEV_TIMEOUT)) {
            *abort = 1;
            return;
        }
        if ((int64_t)(global_timer_ns() - t0) > 2000000000LL) {
            *abort = 1;
            if (status) atomicOr(status, LI_DEV_TIMEOUT);
            return;
        }
    }
}

// M = tensor-core rows (heads, zero-padded to 64 when N1 < 64); C > 1: a
// cluster of C CTAs shares one row, CTA `part` taking its share of the row's
// key tiles; the C partial (max, sum, O) triples are merged through
// distributed shared memory, so no global scratch is needed.
template <int M, bool F16, int C>
__global__ void __launch_bounds__(kThreads, M == 64 ? 2 : 1) sfa_kernel(const SfaArgs a)
{
    using L = Layout<M>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint32_t *sMask = reinterpret_cast<uint32_t *>(base + L::MASK);
    uint64_t *bars = reinterpret_cast<uint64_t *>(base + L::BARS);
    uint64_t *kfull = bars, *kempty = bars + kKStages;
    uint64_t *vfull = bars + 2 * kKStages, *vempty = vfull + kVStages;
    uint64_t *sfull = vempty + kVStages, *sfree = sfull + 2;
    uint64_t *pfull = sfree + 2, *pvdone = pfull + 1;     // the weights buffer
    uint64_t *mfull = pvdone + 1;                         // [kMaskRing]
    uint32_t *tslot = reinterpret_cast<uint32_t *>(base + L::TSLOT);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(base + L::TSLOT + 4);
    const uint32_t sbase = smem_u32(base);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int row = blockIdx.x / C;
    const int part = C > 1 ? (int)(blockIdx.x % C) : 0;   // rank in the cluster

    // ---- the row's batch, its position and the batch's keys
    int b = 0, i = 0, Sq = 0;
    if (a.layout_q == LI_BSND) {
        b = row / a.S1;
        i = row - b * a.S1;
        Sq = a.act_q ? clampi(a.act_q[b], 0, a.S1) : a.S1;
    } else {                                   // prefix sums without a leading 0
        int lo = 0, hi = a.B - 1;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (clampi(a.act_q[mid], 0, a.T1) > row) hi = mid;
            else lo = mid + 1;
        }
        b = lo;
        const int start = b ? clampi(a.act_q[b - 1], 0, a.T1) : 0;
        const int end = clampi(a.act_q[b], start, a.T1);
        i = row - start;
        Sq = end - start;
    }
    int Sk = 0;
    int64_t k_off = 0;
    if (a.layout_kv == LI_BSND) {
        Sk = a.act_k ? clampi(a.act_k[b], 0, a.S2) : a.S2;
        k_off = (int64_t)b * a.S2;
    } else if (a.layout_kv == LI_TND) {
        const int start = b ? clampi(a.act_k[b - 1], 0, a.T2) : 0;
        Sk = clampi(a.act_k[b], start, a.T2) - start;
        k_off = start;
    } else {
        Sk = clampi(a.act_k[b], 0, (int64_t)a.max_blocks_per_seq * a.block_size);
    }
    const bool valid_row = i >= 0 && i < Sq;      // uniform over the CTA
    const int nt_all = valid_row ? (a.K + kSlots - 1) / kSlots : 0;
    const int t_begin = nt_all * part / C, t_end = nt_all * (part + 1) / C;
    const int ntl = t_end - t_begin;              // this CTA's tiles

    if (tid == 0) {
        for (int s = 0; s < kKStages; ++s) {
            mbar_init(&kfull[s], kProducers);     // every producer thread's copies
            mbar_init(&kempty[s], 1);             // the S commit
        }
        for (int s = 0; s < kVStages; ++s) {
            mbar_init(&vfull[s], kProducers);     // every producer thread's copies
            mbar_init(&vempty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sfull[s], 1);
            mbar_init(&sfree[s], 4);
        }
        mbar_init(pfull, 4);                      // the four softmax warps
        mbar_init(pvdone, 1);                     // the P.V commit
        for (int s = 0; s < kMaskRing; ++s) mbar_init(&mfull[s], 2);   // lane 0 of each producer warp
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    if (warp == 2) tmem_alloc(tslot, 256);        // S: two buffers of 64 columns; O: 128-255
    // the producers' slot resolution (thread p of warps 0-1 owns slot p); the
    // first tiles' index loads, and the first block-table load, are issued
    // around the query load so their latencies overlap it
    const int32_t *irow = a.idx + (int64_t)row * a.K;
    const int sp = tid;                           // slot of this thread
    const bool pa = a.layout_kv == LI_PA_BSND;
    const int64_t bt_row = (int64_t)b * a.max_blocks_per_seq;
    auto load_idx = [&](int t) -> int {           // index of this slot in tile t (or -1)
        const int j = t * kSlots + sp;
        return (t < t_end && j < a.K) ? irow[j] : -1;
    };
    auto load_blk = [&](int e) -> int {           // block id behind a valid index
        return (pa && e >= 0 && e < Sk) ? a.block_table[bt_row + (a.bs_shift >= 0 ? e >> a.bs_shift : e / a.block_size)] : 0;
    };
    auto row_of = [&](int e, int id) -> int {     // key row, or -1 (flags bad entries)
        if (e >= 0 && e < Sk) {
            if (!pa) return (int)(k_off + e);
            if (id >= 0 && id < a.num_blocks)
                return id * a.block_size + (a.bs_shift >= 0 ? e & (a.block_size - 1) : e % a.block_size);
            if (a.status) atomicOr(a.status, LI_DEV_BAD_BLOCK);
            return -1;
        }
        if (e != -1 && a.status) atomicOr(a.status, LI_DEV_BAD_INDEX);
        return -1;
    };
    int e_cur = -1, e_nxt = -1, d_cur = 0;
    if (warp < 2) {
        e_cur = load_idx(t_begin);
        e_nxt = load_idx(t_begin + 1);
    }
    // Q into shared memory (heads beyond N1 are zero rows): every load of
    // this thread is issued before the first store, so the query costs one
    // memory latency
    {
        constexpr int kQIter = (M * 16 + kThreads - 1) / kThreads;
        uint4 qv[kQIter];
#pragma unroll
        for (int k = 0; k < kQIter; ++k) {
            const int e = tid + k * kThreads, r = e >> 4, ch = e & 15;
            qv[k] = make_uint4(0, 0, 0, 0);
            if (e < M * 16 && r < a.N1 && valid_row)
                qv[k] = *reinterpret_cast<const uint4 *>(a.q + ((int64_t)row * a.N1 + r) * kHd + ch * 8);
        }
#pragma unroll
        for (int k = 0; k < kQIter; ++k) {
            const int e = tid + k * kThreads, r = e >> 4, ch = e & 15;
            if (e < M * 16) *reinterpret_cast<uint4 *>(base + L::Q + chunk_off(r, ch, L::QPLANE)) = qv[k];
        }
    }
    if (warp < 2) d_cur = load_blk(e_cur);
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tslot;
    const uint32_t tO = tmem + 128;
    const uint16_t *kv_k = a.k, *kv_v = a.v;

    if (warp < 2) {
        // ------------------------------------------------------------ producers
        // thread p resolves slot p of every tile to its key row (index loads
        // two tiles ahead, block-table loads one tile ahead, so no copy waits
        // on a dependent load); the rows are then copied by half warps, 16
        // threads x 16 bytes covering one 256-byte key or value row per
        // copy instruction (fully used 32-byte sectors), zeros for an empty
        // slot.  Each stage is signalled by the copies themselves: the
        // thread's arrival on the stage's full barrier is deferred by the
        // copy unit until all its earlier copies have landed.
        for (int u = 0; u < ntl; ++u) {
            const int t = t_begin + u;
            const int r = row_of(e_cur, d_cur);
            const int d_nxt = load_blk(e_nxt);   // in flight while this tile's copies are issued
            const int e_far = load_idx(t + 2);
            const unsigned ok = __ballot_sync(0xffffffffu, r >= 0);
            int rr[16];                          // rows of slots 32w + 2i + lane/16: one 256-byte row per half warp
#pragma unroll
            for (int i = 0; i < 16; ++i) rr[i] = __shfl_sync(0xffffffffu, r, 2 * i + (lane >> 4));
            const int ks = u % kKStages, vs = u % kVStages;
            // keys of tile u
            wait_phase(&kempty[ks], ((u / kKStages) & 1) ^ 1u, a.status, abort_flag);
            // its validity mask: ring entry u % kMaskRing was last read by the
            // softmax of tile u - kMaskRing, which released its S buffer
            // before S(u - kMaskRing + 2) was issued, which precedes the
            // release of this key stage (kMaskRing >= kKStages + 2)
            if (lane == 0) {
                sMask[(u % kMaskRing) * 2 + warp] = ok;
                mbar_arrive(&mfull[u % kMaskRing]);
            }
            const uint32_t kd = sbase + L::K + ks * kStageBytes;
#pragma unroll
            for (int i = 0; i < 16; ++i)
                cp_async16(kd + chunk_off(32 * warp + 2 * i + (lane >> 4), lane & 15, kPlane),
                           kv_k + (int64_t)(rr[i] < 0 ? 0 : rr[i]) * kHd + (lane & 15) * 8, rr[i] < 0 ? 0u : 16u);
            cp_async_arrive(&kfull[ks]);
            // values of tile u
            wait_phase(&vempty[vs], ((u / kVStages) & 1) ^ 1u, a.status, abort_flag);
            const uint32_t vd = sbase + L::V + vs * kStageBytes;
#pragma unroll
            for (int i = 0; i < 16; ++i)
                cp_async16(vd + chunk_off(32 * warp + 2 * i + (lane >> 4), lane & 15, kPlane),
                           kv_v + (int64_t)(rr[i] < 0 ? 0 : rr[i]) * kHd + (lane & 15) * 8, rr[i] < 0 ? 0u : 16u);
            cp_async_arrive(&vfull[vs]);
            e_cur = e_nxt;
            d_cur = d_nxt;
            e_nxt = e_far;
        }
        cp_async_wait_all();
    } else if (warp == 2) {
        // ------------------------------------------------------------ MMA issuer
        // S(u) is issued one tile ahead of P.V(u-1), so a tile's softmax runs
        // while the previous tile's P.V is on the tensor core
        if (lane == 0 && ntl > 0) {
            const uint32_t fmt = F16 ? 0u : 1u;
            const uint32_t idesc_s = make_idesc(fmt, fmt, M, kSlots);
            const uint32_t idesc_pv = make_idesc(fmt, fmt, M, kHd) | (1u << 16);   // B (values) MN-major
            auto issue_pv = [&](int u) {                 // O += P V of this CTA's tile u
                const int vs = u % kVStages;
                wait_phase(pfull, u & 1, a.status, abort_flag);
                wait_phase(&vfull[vs], (u / kVStages) & 1, a.status, abort_flag);
                fence_proxy_async_smem();        // copies landed by cp.async, read by the tensor core
                tc_fence_after_sync();
                const uint32_t vb = sbase + L::V + vs * kStageBytes;
                const uint32_t pbase = sbase + L::P;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_f16(tO, smem_desc_sw128(pbase + kk * 32),
                            smem_desc_sw128_mn(vb + kk * 16 * 128, kPlane, 1024), idesc_pv,
                            (u > 0 || kk > 0) ? 1u : 0u);
                mma_commit(&vempty[vs]);
                mma_commit(pvdone);
            };
            for (int u = 0; u < ntl; ++u) {
                const int ks = u % kKStages, sb = u & 1;
                wait_phase(&kfull[ks], (u / kKStages) & 1, a.status, abort_flag);
                wait_phase(&sfree[sb], ((u >> 1) & 1) ^ 1u, a.status, abort_flag);
                fence_proxy_async_smem();
                tc_fence_after_sync();
                const uint32_t kb = sbase + L::K + ks * kStageBytes;
#pragma unroll
                for (int c = 0; c < 2; ++c)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_f16(tmem + sb * kSlots, smem_desc_sw128(sbase + L::Q + c * L::QPLANE + kk * 32),
                                smem_desc_sw128(kb + c * kPlane + kk * 32), idesc_s, (c | kk) != 0);
                mma_commit(&sfull[sb]);
                mma_commit(&kempty[ks]);
                if (u > 0) issue_pv(u - 1);
            }
            issue_pv(ntl - 1);
        }
    } else if constexpr (M == 64) {
        // ------------------------------------------------------------ softmax (M = 64)
        // Quarter q's 16 heads sit in lanes 32q..32q+15; read with the
        // 16-lane shape, thread t holds heads 16q + t/4 and 16q + t/4 + 8 and,
        // of each 8-key group j, keys 8j + 2(t%4) and 8j + 2(t%4) + 1; the four
        // threads of a head combine their max and sum with two shuffles.
        const int quarter = warp & 3;
        const uint32_t tlane = (uint32_t)(quarter * 32) << 16;
        const int t0 = lane & 3, t1 = lane >> 2;
        const int hd[2] = {quarter * 16 + t1, quarter * 16 + t1 + 8};
        float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
        for (int u = 0; u < ntl; ++u) {
            const int sb = u & 1;
            wait_phase(&sfull[sb], (u >> 1) & 1, a.status, abort_flag);
            tc_fence_after_sync();
            uint32_t sv[32];
            tmem_ld_16x256b_x8(tmem + sb * kSlots + tlane, sv);
            tmem_ld_wait();
            wait_phase(&mfull[u % kMaskRing], (u / kMaskRing) & 1, a.status, abort_flag);
            const uint32_t mk0 = sMask[(u % kMaskRing) * 2], mk1 = sMask[(u % kMaskRing) * 2 + 1];
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sfree[sb]);   // S buffer (and mask entry) read
            // empty slots get a raw score of -inf (a tile with every slot
            // filled skips the test); the scale is positive, so the max is
            // taken on raw scores and scaled once
            if ((mk0 & mk1) != 0xffffffffu) {
#pragma unroll
                for (int j = 0; j < 8; ++j)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int key = 8 * j + 2 * t0 + (e & 1);
                        if (!(((key < 32 ? mk0 : mk1) >> (key & 31)) & 1u)) sv[4 * j + e] = 0xff800000u;
                    }
            }
            float mx[2], alpha[2], mb[2];
#pragma unroll
            for (int g = 0; g < 2; ++g) {
                auto s_ = [&](int k) { return __uint_as_float(sv[4 * (k >> 1) + 2 * g + (k & 1)]); };
                const float a0 = fmax3(s_(0), s_(1), s_(2)), a1 = fmax3(s_(3), s_(4), s_(5));
                const float a2 = fmax3(s_(6), s_(7), s_(8)), a3 = fmax3(s_(9), s_(10), s_(11));
                const float a4 = fmax3(s_(12), s_(13), s_(14));
                mx[g] = fmaxf(fmax3(a0, a1, a2), fmax3(a3, a4, s_(15)));
                mx[g] = fmaxf(mx[g], __shfl_xor_sync(0xffffffffu, mx[g], 1));
                mx[g] = fmaxf(mx[g], __shfl_xor_sync(0xffffffffu, mx[g], 2));
                mx[g] *= a.scale_log2;
                // move the running max only when this tile beats it by more than 2^8
                alpha[g] = 1.f;
                if (mx[g] > m_run[g] + kRescaleLog2 || (m_run[g] == -INFINITY && mx[g] > -INFINITY)) {
                    alpha[g] = m_run[g] == -INFINITY ? 0.f : ex2(m_run[g] - mx[g]);
                    m_run[g] = mx[g];
                }
                mb[g] = m_run[g] == -INFINITY ? 0.f : -m_run[g];
            }
            // weights exp2(scale_log2 * s - m), two keys per packed fma
            uint32_t pk[16];                      // [j][head]: keys 8j+2t0, +1
            float rs[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
            for (int j = 0; j < 8; ++j)
#pragma unroll
                for (int g = 0; g < 2; ++g) {
                    float x0, x1;
                    ffma2(x0, x1, __uint_as_float(sv[4 * j + 2 * g]), __uint_as_float(sv[4 * j + 2 * g + 1]),
                          a.scale_log2, a.scale_log2, mb[g], mb[g]);
                    const uint32_t w = pack2<F16>(ex2(x0), ex2(x1));
                    pk[2 * j + g] = w;
                    fadd2(rs[g][0], rs[g][1], unpack_lo<F16>(w), unpack_hi<F16>(w));
                }
#pragma unroll
            for (int g = 0; g < 2; ++g) {
                float r = rs[g][0] + rs[g][1];
                r += __shfl_xor_sync(0xffffffffu, r, 1);
                r += __shfl_xor_sync(0xffffffffu, r, 2);
                l_run[g] = l_run[g] * alpha[g] + r;
            }
            // the weights buffer was last read by P.V(u-1), which also
            // completes O for the rescale below
            if (u > 0) {
                wait_phase(pvdone, (u - 1) & 1, a.status, abort_flag);
                tc_fence_after_sync();
            }
            uint8_t *pbuf = base + L::P;
#pragma unroll
            for (int j = 0; j < 8; ++j)
#pragma unroll
                for (int g = 0; g < 2; ++g)
                    *reinterpret_cast<uint32_t *>(pbuf + hd[g] * 128 + ((j ^ (hd[g] & 7)) << 4) + 4 * t0) = pk[2 * j + g];
            // O *= alpha where some head of this warp moved its max (O holds the
            // previous tiles once P.V(u-1) is done; the first tile's P.V
            // overwrites it)
            if (u > 0 && __any_sync(0xffffffffu, alpha[0] != 1.f || alpha[1] != 1.f)) {
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    uint32_t o[32];
                    tmem_ld_16x256b_x8(tO + tlane + 64 * c, o);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha[(e >> 1) & 1]);
                    tmem_st_16x256b_x8(tO + tlane + 64 * c, o);
                }
                tmem_st_wait();
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(pfull);
        }
        if (ntl > 0) {
            // the last P.V (its buffer's latest phase; waiting on a phase that
            // has already completed returns at once)
            wait_phase(pvdone, (ntl - 1) & 1, a.status, abort_flag);
            tc_fence_after_sync();
        }
        // ---- normalise and store (zeros and -inf when nothing was selected)
        const float ln2 = 0.69314718055994531f;
        float *sO = reinterpret_cast<float *>(base + L::K);              // [M][128], unnormalised (C > 1)
        float *sM = reinterpret_cast<float *>(base + L::MERGE);
        float *sL = sM + 128;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            uint32_t o[32];                       // columns 64c + 8j + 2t0 (+1) of heads hd[0], hd[1]
            if (ntl > 0) {
                tmem_ld_16x256b_x8(tO + tlane + 64 * c, o);
                tmem_ld_wait();
            }
#pragma unroll
            for (int j = 0; j < 8; ++j)
#pragma unroll
                for (int g = 0; g < 2; ++g) {
                    const int col = 64 * c + 8 * j + 2 * t0;
                    const float o0 = ntl > 0 ? __uint_as_float(o[4 * j + 2 * g]) : 0.f;
                    const float o1 = ntl > 0 ? __uint_as_float(o[4 * j + 2 * g + 1]) : 0.f;
                    if constexpr (C == 1) {
                        if (hd[g] < a.N1) {
                            const float inv = l_run[g] > 0.f ? 1.f / l_run[g] : 0.f;
                            *reinterpret_cast<uint32_t *>(a.out + ((int64_t)row * a.N1 + hd[g]) * kHd + col) =
                                l_run[g] > 0.f ? pack2<F16>(o0 * inv, o1 * inv) : 0u;
                        }
                    } else {
                        sO[hd[g] * kHd + col] = o0;
                        sO[hd[g] * kHd + col + 1] = o1;
                    }
                }
        }
        if (t0 == 0) {
#pragma unroll
            for (int g = 0; g < 2; ++g) {
                if constexpr (C == 1) {
                    if (a.lse && hd[g] < a.N1)
                        a.lse[(int64_t)row * a.N1 + hd[g]] =
                            l_run[g] > 0.f ? (m_run[g] + log2f(l_run[g])) * ln2 : -INFINITY;
                } else {
                    sM[hd[g]] = m_run[g];
                    sL[hd[g]] = l_run[g];
                }
            }
        }
    } else {
        // ------------------------------------------------------------ softmax (M = 128)
        const int quarter = warp & 3;             // tensor-memory lane quarter of this warp
        const uint32_t tlane = (uint32_t)(quarter * 32) << 16;
        // this thread's head: M = 64 keeps rows 16q..16q+15 in lanes 32q..32q+15
        // of quarter q, M = 128 row r in lane r
        const int h = M == 64 ? (lane < 16 ? quarter * 16 + lane : -1) : quarter * 32 + lane;
        float m_run = -INFINITY, l_run = 0.f;     // log2-domain running max and sum
        for (int u = 0; u < ntl; ++u) {
            const int sb = u & 1;
            wait_phase(&sfull[sb], (u >> 1) & 1, a.status, abort_flag);
            tc_fence_after_sync();
            uint32_t sv[64];
            const uint32_t ts = tmem + sb * kSlots + tlane;
            tmem_ld16_into<0>(ts, sv);
            tmem_ld16_into<1>(ts, sv);
            tmem_ld16_into<2>(ts, sv);
            tmem_ld16_into<3>(ts, sv);
            tmem_ld_wait();
            wait_phase(&mfull[u % kMaskRing], (u / kMaskRing) & 1, a.status, abort_flag);
            const uint32_t mk0 = sMask[(u % kMaskRing) * 2], mk1 = sMask[(u % kMaskRing) * 2 + 1];
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sfree[sb]);   // S buffer (and mask entry) read
            if ((mk0 & mk1) != 0xffffffffu) {     // empty slots: raw score -inf
#pragma unroll
                for (int j = 0; j < 64; ++j)
                    if (!(((j < 32 ? mk0 : mk1) >> (j & 31)) & 1u)) sv[j] = 0xff800000u;
            }
            float mx[22];
#pragma unroll
            for (int j = 0; j < 21; ++j)
                mx[j] = fmax3(__uint_as_float(sv[3 * j]), __uint_as_float(sv[3 * j + 1]), __uint_as_float(sv[3 * j + 2]));
            mx[21] = __uint_as_float(sv[63]);
#pragma unroll
            for (int j = 0; j < 7; ++j) mx[j] = fmax3(mx[3 * j], mx[3 * j + 1], mx[3 * j + 2]);
            const float mt = fmaxf(fmaxf(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5])),
                                   fmaxf(mx[6], mx[21])) * a.scale_log2;
            // move the running max only when this tile beats it by more than 2^8
            float alpha = 1.f;
            if (h >= 0 && (mt > m_run + kRescaleLog2 || (m_run == -INFINITY && mt > -INFINITY))) {
                alpha = m_run == -INFINITY ? 0.f : ex2(m_run - mt);
                m_run = mt;
            }
            const float mb = m_run == -INFINITY ? 0.f : -m_run;
            float rs[4][2] = {};
            uint32_t pk[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                float x0, x1;
                ffma2(x0, x1, __uint_as_float(sv[2 * j]), __uint_as_float(sv[2 * j + 1]), a.scale_log2, a.scale_log2,
                      mb, mb);
                pk[j] = pack2<F16>(ex2(x0), ex2(x1));
                fadd2(rs[j & 3][0], rs[j & 3][1], unpack_lo<F16>(pk[j]), unpack_hi<F16>(pk[j]));
            }
            rs[0][0] += rs[2][0] + (rs[1][0] + rs[3][0]);
            rs[0][1] += rs[2][1] + (rs[1][1] + rs[3][1]);
            rs[0][0] += rs[0][1];
            l_run = l_run * alpha + rs[0][0];
            // the weights buffer was last read by P.V(u-1), which also
            // completes O for the rescale below
            if (u > 0) {
                wait_phase(pvdone, (u - 1) & 1, a.status, abort_flag);
                tc_fence_after_sync();
            }
            if (h >= 0) {
#pragma unroll
                for (int ch = 0; ch < 8; ++ch)
                    *reinterpret_cast<uint4 *>(base + L::P + chunk_off(h, ch, L::QPLANE)) =
                        make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
            }
            // O *= alpha where some head of this warp moved its max (O holds the
            // previous tiles once P.V(u-1) is done; the first tile's P.V
            // overwrites it)
            const bool rescale = u > 0 && __any_sync(0xffffffffu, alpha != 1.f);
            if (rescale) {
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    uint32_t o16[16];
                    tmem_ld16(tO + tlane + 16 * c, o16);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 16; ++e) o16[e] = __float_as_uint(__uint_as_float(o16[e]) * alpha);
                    tmem_st16(tO + tlane + 16 * c, o16);
                }
                tmem_st_wait();
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(pfull);
        }
        if (ntl > 0) {
            // the last P.V (its buffer's latest phase; waiting on a phase that
            // has already completed returns at once)
            wait_phase(pvdone, (ntl - 1) & 1, a.status, abort_flag);
            tc_fence_after_sync();
        }
        // ---- normalise and store (zeros and -inf when nothing was selected)
        if constexpr (C == 1) {
            const float ln2 = 0.69314718055994531f;
            const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
            uint16_t *orow = a.out + ((int64_t)row * a.N1 + (h < 0 ? 0 : h)) * kHd;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint32_t o16[16];
                if (ntl > 0) {
                    tmem_ld16(tO + tlane + 16 * c, o16);
                    tmem_ld_wait();
                }
                if (h >= 0 && h < a.N1) {
                    uint32_t w8[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        w8[e] = ntl > 0 && l_run > 0.f
                                    ? pack2<F16>(__uint_as_float(o16[2 * e]) * inv, __uint_as_float(o16[2 * e + 1]) * inv)
                                    : 0u;
                    *reinterpret_cast<uint4 *>(orow + 16 * c) = make_uint4(w8[0], w8[1], w8[2], w8[3]);
                    *reinterpret_cast<uint4 *>(orow + 16 * c + 8) = make_uint4(w8[4], w8[5], w8[6], w8[7]);
                }
            }
            if (a.lse && h >= 0 && h < a.N1)
                a.lse[(int64_t)row * a.N1 + h] = l_run > 0.f ? (m_run + log2f(l_run)) * ln2 : -INFINITY;
        } else {
            // partials into this CTA's shared memory (the key/value rings are
            // free: every MMA has completed)
            float *sO = reinterpret_cast<float *>(base + L::K);              // [M][128], unnormalised
            float *sM = reinterpret_cast<float *>(base + L::MERGE);          // [128]
            float *sL = sM + 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint32_t o16[16];
                if (ntl > 0) {
                    tmem_ld16(tO + tlane + 16 * c, o16);
                    tmem_ld_wait();
                }
                if (h >= 0)
#pragma unroll
                    for (int e = 0; e < 16; ++e) sO[h * kHd + 16 * c + e] = ntl > 0 ? __uint_as_float(o16[e]) : 0.f;
            }
            if (h >= 0) {
                sM[h] = m_run;
                sL[h] = l_run;
            }
        }
    }

    if constexpr (C > 1) {
        // CTA `part` merges heads [part*N1/C, (part+1)*N1/C) over the C partials
        float *sO = reinterpret_cast<float *>(base + L::K);
        float *sM = reinterpret_cast<float *>(base + L::MERGE);
        float *sL = sM + 128;
        float *sWt = sL + 128;                 // [hpc][C]: each partial's weight exp2(m_r - M) / L
        cooperative_groups::cluster_group cl = cooperative_groups::this_cluster();
        cl.sync();
        const float ln2 = 0.69314718055994531f;
        const int hpc = a.N1 / C;
        // per (head, partial): the merged max and normaliser, then the weight
        // of that partial's unnormalised output
        for (int e = tid; e < hpc * C; e += kThreads) {
            const int hl = e / C, r = e % C, hh = part * hpc + hl;
            float Mx = -INFINITY;
#pragma unroll
            for (int q = 0; q < C; ++q) Mx = fmaxf(Mx, cl.map_shared_rank(sM, q)[hh]);
            float Ls = 0.f;
            if (Mx != -INFINITY) {
#pragma unroll
                for (int q = 0; q < C; ++q) {
                    const float mq = cl.map_shared_rank(sM, q)[hh];
                    if (mq != -INFINITY) Ls += cl.map_shared_rank(sL, q)[hh] * exp2f(mq - Mx);
                }
            }
            const float mr = cl.map_shared_rank(sM, r)[hh];
            sWt[e] = (Ls > 0.f && mr != -INFINITY) ? exp2f(mr - Mx) / Ls : 0.f;
            if (r == 0 && a.lse) a.lse[(int64_t)row * a.N1 + hh] = Ls > 0.f ? (Mx + log2f(Ls)) * ln2 : -INFINITY;
        }
        __syncthreads();
        // out = sum_r weight_r * O_r, four columns per thread and step
        for (int e = tid; e < hpc * (kHd / 4); e += kThreads) {
            const int hl = e / (kHd / 4), d4 = e % (kHd / 4), hh = part * hpc + hl;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int r = 0; r < C; ++r) {
                const float w = sWt[hl * C + r];
                if (w != 0.f) {
                    const float4 o = reinterpret_cast<const float4 *>(cl.map_shared_rank(sO, r))[hh * (kHd / 4) + d4];
                    acc.x += w * o.x;
                    acc.y += w * o.y;
                    acc.z += w * o.z;
                    acc.w += w * o.w;
                }
            }
            *reinterpret_cast<uint2 *>(a.out + ((int64_t)row * a.N1 + hh) * kHd + 4 * d4) =
                make_uint2(pack2<F16>(acc.x, acc.y), pack2<F16>(acc.z, acc.w));
        }
        cl.sync();                             // every peer has read this CTA's partials
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 2) tmem_dealloc(tmem, 256);
}

// Rows when the key tensor is empty: out = 0, lse = -inf.
template <bool F16>
__global__ void sfa_empty_kernel(uint16_t *out, float *lse, int64_t rows, int N1)
{
    const int64_t n = rows * N1 * kHd;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
        out[e] = 0;
        if (lse && e % kHd == 0) lse[e / kHd] = -INFINITY;
    }
}

template <int M, bool F16, int C>
cudaError_t launch(const SfaArgs &a, int rows, cudaStream_t s)
{
    auto kern = sfa_kernel<M, F16, C>;
    const int smem = Layout<M>::BYTES;
    cudaError_t e = li::set_max_dynamic_smem(reinterpret_cast<const void *>(kern), smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)rows * C);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a);
}

template <int M, bool F16>
cudaError_t launch_split(const SfaArgs &a, int rows, int split, cudaStream_t s)
{
    switch (split) {
    case 1: return launch<M, F16, 1>(a, rows, s);
    case 2: return launch<M, F16, 2>(a, rows, s);
    case 4: return launch<M, F16, 4>(a, rows, s);
    case 8: return launch<M, F16, 8>(a, rows, s);
    }
    return cudaErrorInvalidValue;
}

template <bool F16>
cudaError_t launch_m(const SfaArgs &a, int rows, int split, cudaStream_t s)
{
    return a.N1 <= 64 ? launch_split<64, F16>(a, rows, split, s) : launch_split<128, F16>(a, rows, split, s);
}

// CTAs per row when rows are few (decode): the largest power of two up to 8
// that keeps the grid within one wave of two CTAs per SM, with at least four
// 64-key tiles per CTA.
int choose_split(int64_t rows, int K, int sms)
{
    const int ntiles = (K + kSlots - 1) / kSlots;
    int c = 1;
    while (c < kMaxSplit && rows * c * 2 <= 2LL * sms && 4 * c * 2 <= ntiles) c *= 2;
    return c;
}

bool aligned(const void *p, uintptr_t n) { return (reinterpret_cast<uintptr_t>(p) & (n - 1)) == 0; }

}  // namespace

extern "C" LI_API li_status li_sparse_attention(const li_sfa_params *p, const void *query, const void *key,
                                                const void *value, const int32_t *sparse_indices,
                                                const int32_t *act_seq_q, const int32_t *act_seq_k,
                                                const int32_t *block_table, void *out, float *lse,
                                                int32_t *status, void *stream)
{
    using li::report_error;
    if (!p || !query || !key || !value || !sparse_indices || !out)
        return report_error(LI_ERR_NULL, "li_sparse_attention: a required pointer is NULL");
    if (p->reserved != 0) return report_error(LI_ERR_SHAPE, "li_sparse_attention: reserved must be 0");
    if (p->dtype != LI_BF16 && p->dtype != LI_FP16)
        return report_error(LI_ERR_DTYPE, "li_sparse_attention: dtype must be LI_BF16 or LI_FP16");
    if (p->layout_q != LI_BSND && p->layout_q != LI_TND)
        return report_error(LI_ERR_LAYOUT, "li_sparse_attention: layout_q must be BSND or TND");
    if (p->layout_kv != LI_PA_BSND && p->layout_kv != p->layout_q)
        return report_error(LI_ERR_LAYOUT, "li_sparse_attention: layout_kv must equal layout_q or be PA_BSND");
    if (p->N1 != 16 && p->N1 != 32 && p->N1 != 64 && p->N1 != 128)
        return report_error(LI_ERR_SHAPE, "li_sparse_attention: N1 must be 16, 32, 64 or 128");
    if (p->D != kHd || p->Dv != kHd)
        return report_error(LI_ERR_UNSUPPORTED, "li_sparse_attention: D and Dv must be 128");
    if (p->sparse_count < 1 || p->sparse_count > 65536)
        return report_error(LI_ERR_SHAPE, "li_sparse_attention: sparse_count must be in [1, 65536]");
    if (!(p->softmax_scale > 0.f) || !std::isfinite(p->softmax_scale))
        return report_error(LI_ERR_SHAPE, "li_sparse_attention: softmax_scale must be positive and finite");
    if (p->B < 1) return report_error(LI_ERR_SHAPE, "li_sparse_attention: B must be >= 1");
    int64_t rows = 0, key_rows = 0;
    if (p->layout_q == LI_BSND) {
        if (p->S1 < 0) return report_error(LI_ERR_SHAPE, "li_sparse_attention: S1 must be >= 0");
        rows = (int64_t)p->B * p->S1;
    } else {
        if (p->T1 < 0) return report_error(LI_ERR_SHAPE, "li_sparse_attention: T1 must be >= 0");
        if (!act_seq_q) return report_error(LI_ERR_NULL, "li_sparse_attention: TND needs act_seq_q");
        rows = p->T1;
    }
    if (p->layout_kv == LI_BSND) {
        if (p->S2 < 0) return report_error(LI_ERR_SHAPE, "li_sparse_attention: S2 must be >= 0");
        key_rows = (int64_t)p->B * p->S2;
    } else if (p->layout_kv == LI_TND) {
        if (p->T2 < 0) return report_error(LI_ERR_SHAPE, "li_sparse_attention: T2 must be >= 0");
        if (!act_seq_k) return report_error(LI_ERR_NULL, "li_sparse_attention: TND needs act_seq_k");
        key_rows = p->T2;
    } else {
        if (!act_seq_k || !block_table)
            return report_error(LI_ERR_NULL, "li_sparse_attention: PA_BSND needs act_seq_k and block_table");
        if (p->num_blocks < 1 || p->block_size < 1 || p->max_blocks_per_seq < 1)
            return report_error(LI_ERR_SHAPE, "li_sparse_attention: PA pool dimensions must be >= 1");
        key_rows = (int64_t)p->num_blocks * p->block_size;
    }
    if (rows > 0x7FFFFFFF || key_rows > 0x7FFFFFFF || (int64_t)p->max_blocks_per_seq * p->block_size > 0x7FFFFFFF)
        return report_error(LI_ERR_SHAPE, "li_sparse_attention: more than 2^31-1 query or key rows");
    if (!aligned(query, 16) || !aligned(key, 16) || !aligned(value, 16) || !aligned(out, 16) ||
        !aligned(sparse_indices, 4) || (lse && !aligned(lse, 4)) || (status && !aligned(status, 4)))
        return report_error(LI_ERR_SHAPE, "li_sparse_attention: query/key/value/out must be 16-byte aligned, "
                                          "sparse_indices/lse/status 4-byte aligned");
    li::set_launch_count(0);
    if (rows == 0) return LI_OK;
    SfaArgs a{};
    a.q = static_cast<const uint16_t *>(query);
    a.k = static_cast<const uint16_t *>(key);
    a.v = static_cast<const uint16_t *>(value);
    a.idx = sparse_indices;
    a.act_q = act_seq_q;
    a.act_k = act_seq_k;
    a.block_table = block_table;
    a.out = static_cast<uint16_t *>(out);
    a.lse = lse;
    a.status = status;
    a.layout_q = p->layout_q;
    a.layout_kv = p->layout_kv;
    a.B = p->B;
    a.S1 = p->S1;
    a.S2 = p->S2;
    a.T1 = p->T1;
    a.T2 = p->T2;
    a.N1 = p->N1;
    a.K = p->sparse_count;
    a.num_blocks = p->num_blocks;
    a.block_size = p->block_size;
    a.max_blocks_per_seq = p->max_blocks_per_seq;
    a.scale_log2 = p->softmax_scale * 1.4426950408889634f;
    a.bs_shift = -1;
    if (p->block_size > 0 && (p->block_size & (p->block_size - 1)) == 0) {
        a.bs_shift = 0;
        while ((1 << a.bs_shift) < p->block_size) ++a.bs_shift;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaError_t e;
    if (key_rows == 0) {
        // no key can be selected: every row is empty
        const int grid = (int)((rows * p->N1 * kHd + 255) / 256 < 4096 ? (rows * p->N1 * kHd + 255) / 256 : 4096);
        if (p->dtype == LI_FP16)
            sfa_empty_kernel<true><<<grid, 256, 0, s>>>(a.out, a.lse, rows, p->N1);
        else
            sfa_empty_kernel<false><<<grid, 256, 0, s>>>(a.out, a.lse, rows, p->N1);
        e = cudaGetLastError();
    } else {
        const int split = choose_split(rows, a.K, sms);
        e = p->dtype == LI_FP16 ? launch_m<true>(a, (int)rows, split, s) : launch_m<false>(a, (int)rows, split, s);
    }
    if (e != cudaSuccess) {
        char msg[200];
        snprintf(msg, sizeof msg, "li_sparse_attention: launch failed (%s)", cudaGetErrorString(e));
        return report_error(LI_ERR_CUDA, msg);
    }
    li::set_launch_count(1);
    return LI_OK;
}
