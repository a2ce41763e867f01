// li_score.cu -- the fused score kernel: s(t) for every visible (query, key).
//
// Computes, per query token i and key t (mindspore.ops.lightning_indexer page,
// ".. math::"; CANN LightningIndexerV2 guide, "三步计算流程"; for fp8 the
// VllmQuantLightningIndexer README, "功能说明"):
//
//     s(i,t) = [Scale_K(t) *] sum_h [W(i,h) * Scale_Q(i,h)] * ReLU(q(i,h) . k(t))
//
// (for scales >= 0 this equals sum_h W * ReLU(Scale_Q * Scale_K * q.k), the
// README's order) and stores it, for the keys the sparse mode leaves visible,
// into one fp32 score row per query.  Per-head logits never leave the SM.
//
// Design (one persistent CTA per SM, warp-specialised):
//   warp 0     TMA producer: loads the query block (all heads of up to
//              256/N1P queries, K-major, 128-byte swizzle) once per block and
//              streams 128-key tiles through a STAGES-deep ring; paged keys
//              are gathered block by block through block_table.
//   warp 1     allocates 512 TMEM columns and issues tcgen05.mma
//              (M = 128 keys, N = queries*heads <= 256, K = D) into one of two
//              fp32 TMEM accumulators, then commits to the ring / accumulator
//              barriers.
//   warps 2-17 epilogue, two groups of eight, one per accumulator (group g
//              takes every other tile): each thread owns one key (one TMEM
//              lane), streams that lane's head columns out of TMEM 16 at a
//              time (double-buffered, the accumulator handed back once the
//              last chunk is in registers) and reduces them in registers --
//              ReLU, multiply by the weight, sum over heads, scale -- then
//              writes the score if the key is visible.
// Work is a flat list of (query block, key tile) units written by the
// device-side scheduler; each CTA takes a contiguous, equal share, so causal
// triangles and ragged lengths are balanced over the SMs.
#include <cstdint>
#include <cuda_fp16.h>

#include "li_internal.cuh"
#include "ptx.cuh"

namespace li {
namespace {

constexpr int kRowBytes = 128;                        // one swizzle row
constexpr int kQRows = 256;

template <int CHUNKS>
struct Geometry {
    static constexpr int STAGES = CHUNKS == 2 ? 4 : 6;
    static constexpr int Q_BYTES = kQRows * kRowBytes * CHUNKS;
    static constexpr int Q_CHUNK = kQRows * kRowBytes;
    static constexpr int K_CHUNK = kTileKeys * kRowBytes;
    static constexpr int K_BYTES = K_CHUNK * CHUNKS;
    static constexpr int W_FLOATS = kEpiWarps * 128;
    static constexpr int NBARS = 2 * STAGES + 7;
    static constexpr int TABLE = 1024;         // block_table entries of one batch staged in smem
    static constexpr size_t SMEM = 1024 + Q_BYTES + (size_t)STAGES * K_BYTES + W_FLOATS * 4 +
                                   TABLE * 4 + NBARS * 8 + 16;
};

// Walks this CTA's share [w0, w1) of the weighted work list.  A block of n
// key tiles occupies n + q_cost consecutive positions: q_cost for loading its
// query tile, then one per key tile; a tile belongs to the CTA whose range
// holds its position, so every tile is processed exactly once.
struct Walker {
    const BlockInfo *blocks;
    int nblocks, w_end, qcost;
    int qb, tile, ntiles, start;
    __device__ void load_block()
    {
        if (qb < nblocks) {
            start = blocks[qb].unit_start;
            ntiles = blocks[qb].ntiles;
        }
    }
    __device__ void normalize()
    {
        while (qb < nblocks && tile >= ntiles) {
            ++qb;
            tile = 0;
            load_block();
        }
    }
    // start at the scheduler's record of where this CTA's share [w0, w1)
    // begins: the last block starting at or before w0, the tile inside it,
    // moved past blocks without a tile in the share
    __device__ void init_from(const int4 st, int w1)
    {
        w_end = w1;
        qb = st.x;
        tile = st.y;
        start = st.z;
        ntiles = st.w;
    }
    __device__ bool valid() const { return qb < nblocks && start + qcost + tile < w_end; }
    __device__ void next()
    {
        ++tile;
        normalize();
    }
};

__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

__device__ __forceinline__ uint64_t pack2(float lo, float hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ void unpack2(uint64_t r, float &lo, float &hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(r));
}

__device__ __forceinline__ float hsum2(uint64_t r)
{
    float lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(r));
    return lo + hi;
}


// ReLU, split over two pipes.  max(x, 0) runs on the ALU pipe at half the
// FP32 rate; x + |x| = 2*ReLU(x) exactly is one FADD on the FMA pipe, with the
// factor 1/2 folded into that column's weight (a power-of-two scaling, so the
// product W*ReLU(x) rounds the same).  Three of every eight columns take the
// FADD form, which balances the two pipes against the packed FMAs.
constexpr int kFaddPer8 = 3;
__host__ __device__ constexpr bool fadd_col(int col) { return (col & 7) < kFaddPer8; }

template <int COL>
__device__ __forceinline__ float relu_c(float x)
{
    if constexpr (fadd_col(COL)) return x + fabsf(x);
    else return fmaxf(x, 0.f);
}

// Four columns COL0..COL0+3 of the warp's 128: W * ReLU(logit) accumulated
// into the packed partial sums of their query.
template <int COL0, int QPW, int NP2, int N1P>
__device__ __forceinline__ void epi_quad(const float *v, const uint4 ww, uint64_t (&part)[QPW][NP2])
{
    constexpr int q = COL0 / N1P;
    constexpr int p0 = (COL0 / 2) % NP2, p1 = (COL0 / 2 + 1) % NP2;
    const uint64_t w01 = pack2(__uint_as_float(ww.x), __uint_as_float(ww.y));
    const uint64_t w23 = pack2(__uint_as_float(ww.z), __uint_as_float(ww.w));
    part[q][p0] = ffma2(w01, pack2(relu_c<COL0>(v[0]), relu_c<COL0 + 1>(v[1])), part[q][p0]);
    part[q][p1] = ffma2(w23, pack2(relu_c<COL0 + 2>(v[2]), relu_c<COL0 + 3>(v[3])), part[q][p1]);
}

// s32 accumulator bits to fp32, in place; exact for |x| < 2^22 (an int8 dot
// product over D = 128 is at most 2^21): the bit pattern of 1.5*2^23 plus x
// is the float 1.5*2^23 + x, and subtracting 1.5*2^23 leaves x.
__device__ __forceinline__ void s32_to_f32_16(uint32_t (&r)[16])
{
    const uint64_t m2 = pack2(-12582912.f, -12582912.f);
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
        float lo, hi;
        unpack2(fadd2(pack2(__uint_as_float(r[i] + 0x4B400000u), __uint_as_float(r[i + 1] + 0x4B400000u)), m2), lo, hi);
        r[i] = __float_as_uint(lo);
        r[i + 1] = __float_as_uint(hi);
    }
}

__device__ __forceinline__ void release_acc(uint64_t *bar, int lane)
{
    tc_fence_before_sync();
    __syncwarp();
    if (lane == 0) mbar_arrive(bar);
}

// 16-column chunk C of the warp's 128 columns.  The chunk's TMEM load was
// issued into `cur` by the previous step; this step waits for it, issues the
// next chunk's load into `nxt` (or, after the last load, hands the
// accumulator back to the MMA warp), then reduces `cur` while the next load
// is in flight.
template <int C, int QPW, int NP2, int N1P, int KIND>
__device__ __forceinline__ void epi_step(uint32_t trow, int nc, const float *myW,
                                         uint64_t (&part)[QPW][NP2], uint64_t *bar, int lane,
                                         uint32_t (&cur)[16], uint32_t (&nxt)[16])
{
    if constexpr (C < 8) {
        if (C >= nc) return;
        tmem_ld_wait16(cur);
        if (C + 1 < nc) tmem_ld16(trow + 16 * (C + 1), nxt);
        else release_acc(bar, lane);
        if constexpr (KIND == kKindI8) s32_to_f32_16(cur);
        const float *v = reinterpret_cast<const float *>(cur);
        const uint4 *w4 = reinterpret_cast<const uint4 *>(myW + C * 16);
        epi_quad<C * 16 + 0, QPW, NP2, N1P>(v + 0, w4[0], part);
        epi_quad<C * 16 + 4, QPW, NP2, N1P>(v + 4, w4[1], part);
        epi_quad<C * 16 + 8, QPW, NP2, N1P>(v + 8, w4[2], part);
        epi_quad<C * 16 + 12, QPW, NP2, N1P>(v + 12, w4[3], part);
        epi_step<C + 1, QPW, NP2, N1P, KIND>(trow, nc, myW, part, bar, lane, nxt, cur);
    }
}

// Reduces the warp's columns (nc 16-column chunks, nc >= 1) into `part`,
// double-buffering the TMEM loads; the accumulator is released as soon as
// the last chunk is in registers.
template <int QPW, int NP2, int N1P, int KIND>
__device__ __forceinline__ void epi_reduce(uint32_t trow, int nc, const float *myW,
                                           uint64_t (&part)[QPW][NP2], uint64_t *bar, int lane)
{
    uint32_t b0[16], b1[16];
    tmem_ld16(trow, b0);
    epi_step<0, QPW, NP2, N1P, KIND>(trow, nc, myW, part, bar, lane, b0, b1);
}

__device__ __forceinline__ float load_weight(const void *w, int dtype, int64_t i)
{
    if (dtype == LI_FP32) return static_cast<const float *>(w)[i];
    const unsigned short h = static_cast<const unsigned short *>(w)[i];
    if (dtype == LI_BF16) return __uint_as_float((uint32_t)h << 16);
    return __half2float(__ushort_as_half(h));
}

__device__ __forceinline__ float load_scale(const void *p, int dtype, int64_t i)
{
    if (dtype == LI_FP32) return static_cast<const float *>(p)[i];
    return __half2float(__ushort_as_half(static_cast<const unsigned short *>(p)[i]));
}

__device__ __forceinline__ void fail(PlanHeader *hdr, volatile int *abort_flag, int bit)
{
    atomicOr(&hdr->status, bit);
    *abort_flag = 1;
}

template <int CHUNKS, int N1P, int KIND>
__global__ void __launch_bounds__(kScoreThreads, 1)
    score_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                 const ScoreArgs a)
{
    using G = Geometry<CHUNKS>;
    constexpr int STAGES = G::STAGES;
    constexpr int NQ = 256 / N1P;                 // queries per block
    constexpr int QPW = 128 / N1P;                // queries per epilogue warp half
    constexpr int NP2 = N1P >= 64 ? 4 : (N1P == 32 ? 2 : 1);  // packed partial sums per query
    constexpr int INNER = KIND == kKindF16 ? 64 : 128;   // elements per 128-byte row chunk

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem;
    uint8_t *sK = smem + G::Q_BYTES;
    float *sW = reinterpret_cast<float *>(sK + STAGES * G::K_BYTES);
    int32_t *sTable = reinterpret_cast<int32_t *>(sW + G::W_FLOATS);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sTable + G::TABLE);
    uint64_t *k_full = bars;
    uint64_t *k_empty = bars + STAGES;
    uint64_t *q_full = bars + 2 * STAGES;
    uint64_t *q_empty = q_full + 1;
    uint64_t *acc_full = q_full + 2;
    uint64_t *acc_empty = q_full + 4;
    uint64_t *drain = q_full + 6;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + G::NBARS);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
        }
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int s = 0; s < kAccStages; ++s) {
            mbar_init(&acc_full[s], 1);
            mbar_init(&acc_empty[s], kGroupWarps);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    if (a.q_box_rows != kQRows) {
        // per-query Q boxes leave the padded head rows untouched: zero them once
        uint4 *q4 = reinterpret_cast<uint4 *>(sQ);
        for (int j = tid; j < G::Q_BYTES / 16; j += kScoreThreads) q4[j] = make_uint4(0, 0, 0, 0);
        fence_proxy_async_smem();
    }
    if (warp == 1) tmem_alloc(tmem_slot, 2 * kAccCols);
    if (tid == 0) {
        tma_prefetch_desc(&qmap);
        tma_prefetch_desc(&kmap);
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;
    // the prologue above overlaps the scheduler's tail; its work list is read below
    grid_dependency_wait();
    grid_launch_dependents();

    const int total = a.hdr->total_units;
    const int nblocks = a.hdr->total_blocks;
    const int w_begin = (int)(((int64_t)total * blockIdx.x) / gridDim.x);
    const int w_end = (int)(((int64_t)total * (blockIdx.x + 1)) / gridDim.x);

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        // The whole warp walks the work list; lane 0 waits on the ring and
        // issues the copies.  For paged keys the warp stages the batch's
        // block_table row in shared memory at each block switch, so the
        // per-tile block lookups are shared-memory reads, not dependent
        // global loads on the copy path.
        if (w_begin < w_end && nblocks > 0) {
            Walker w{a.blocks, nblocks, 0, a.q_cost, 0, 0, 0, 0};
            w.init_from(a.cta_start[blockIdx.x], w_end);
            int stage = 0, prev_qb = -1;
            uint32_t phase = 0, qphase = 0;
            uint32_t armed = 0, par = 0, q_armed = 0, q_par = 0;
            BlockInfo blk{};
            BatchInfo bi{};
            bool table_in_smem = false;
            int ok = 1;
            for (; w.valid(); w.next()) {
                if (w.qb != prev_qb) {
                    blk = a.blocks[w.qb];
                    bi = a.batches[blk.b];
                    if (a.is_pa) {
                        const int need = (bi.Sk + a.block_size - 1) / a.block_size;
                        table_in_smem = need <= G::TABLE;
                        __syncwarp();
                        if (table_in_smem) {
                            const int32_t *row = a.block_table + (int64_t)blk.b * a.max_blocks_per_seq;
                            for (int j = lane; j < need; j += 32) sTable[j] = row[j];
                        }
                        __syncwarp();
                    }
                    if (lane == 0) {
                        if (!mbar_wait_bounded(q_empty, qphase ^ 1u, abort_flag, a.timeout_ns)) {
                            fail(a.hdr, abort_flag, LI_DEV_TIMEOUT);
                            ok = 0;
                        } else {
                            const int qrow0 = bi.q_off + blk.i0;
                            if (a.q_box_rows == kQRows) {
                                mbar_arrive_expect_tx(q_full, CHUNKS * G::Q_CHUNK);
                                if (a.q_single)
                                    tma_load_3d(sQ, &qmap, q_full, 0, qrow0 * a.N1, 0);
                                else
                                    for (int c = 0; c < CHUNKS; ++c)
                                        tma_load_2d(sQ + c * G::Q_CHUNK, &qmap, q_full, c * INNER,
                                                    qrow0 * a.N1);
                            } else {
                                mbar_arrive_expect_tx(q_full, CHUNKS * NQ * a.N1 * kRowBytes);
                                for (int qi = 0; qi < NQ; ++qi)
                                    for (int c = 0; c < CHUNKS; ++c)
                                        tma_load_2d(sQ + c * G::Q_CHUNK + qi * N1P * kRowBytes, &qmap,
                                                    q_full, c * INNER, (qrow0 + qi) * a.N1);
                            }
                            q_armed = 1;
                            q_par = qphase;
                            qphase ^= 1u;
                        }
                    }
                    if (!__shfl_sync(0xffffffffu, ok, 0)) break;
                    prev_qb = w.qb;
                }
                if (lane == 0) {
                    if (!mbar_wait_bounded(&k_empty[stage], phase ^ 1u, abort_flag, a.timeout_ns)) {
                        fail(a.hdr, abort_flag, LI_DEV_TIMEOUT);
                        ok = 0;
                    } else {
                        uint8_t *dst = sK + stage * G::K_BYTES;
                        const int t0 = w.tile * kTileKeys;
                        if (!a.is_pa) {
                            mbar_arrive_expect_tx(&k_full[stage], G::K_BYTES);
                            if (a.k_single)
                                tma_load_3d(dst, &kmap, &k_full[stage], 0, bi.k_off + t0, 0);
                            else
                                for (int c = 0; c < CHUNKS; ++c)
                                    tma_load_2d(dst + c * G::K_CHUNK, &kmap, &k_full[stage],
                                                c * INNER, bi.k_off + t0);
                        } else {
                            // gather the tile from the paged pool, g = pa_box_rows keys at a time
                            const int g = a.pa_box_rows, nseg = kTileKeys / g;
                            int blkid[8];
                            int nvalid = 0;
                            for (int s = 0; s < nseg; ++s) {
                                const int t = t0 + s * g;
                                blkid[s] = -1;
                                if (t >= bi.Sk) continue;
                                const int lb = t / a.block_size;
                                const int id = table_in_smem
                                                   ? sTable[lb]
                                                   : a.block_table[(int64_t)blk.b * a.max_blocks_per_seq + lb];
                                if (id < 0 || id >= a.num_blocks) {
                                    atomicOr(&a.hdr->status, LI_DEV_BAD_BLOCK);
                                    continue;
                                }
                                blkid[s] = id;
                                ++nvalid;
                            }
                            mbar_arrive_expect_tx(&k_full[stage], nvalid * g * kRowBytes * CHUNKS);
                            for (int s = 0; s < nseg; ++s) {
                                if (blkid[s] < 0) continue;
                                const int t = t0 + s * g;
                                if (a.k_single)             // g == 128: the whole tile, both chunks
                                    tma_load_4d(dst, &kmap, &k_full[stage], 0, t % a.block_size, 0,
                                                blkid[s]);
                                else
                                    for (int c = 0; c < CHUNKS; ++c)
                                        tma_load_3d(dst + c * G::K_CHUNK + s * g * kRowBytes, &kmap,
                                                    &k_full[stage], c * INNER, t % a.block_size,
                                                    blkid[s]);
                            }
                        }
                        armed |= 1u << stage;
                        par = (par & ~(1u << stage)) | (phase << stage);
                        if (++stage == STAGES) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                }
                if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            }
            if (lane == 0 && *abort_flag) {
                // let every copy still in flight land before the CTA exits
                for (int s = 0; s < STAGES; ++s)
                    if (armed & (1u << s))
                        mbar_wait_bounded(&k_full[s], (par >> s) & 1u, nullptr, a.timeout_ns);
                if (q_armed) mbar_wait_bounded(q_full, q_par, nullptr, a.timeout_ns);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && w_begin < w_end && nblocks > 0) {
            Walker w{a.blocks, nblocks, 0, a.q_cost, 0, 0, 0, 0};
            w.init_from(a.cta_start[blockIdx.x], w_end);
            int stage = 0, acc = 0, prev_qb = -1;
            uint32_t phase = 0, acc_phase = 0, qphase = 0, idesc = 0;
            bool issued = false;
            const uint32_t sQ_addr = smem_u32(sQ), sK_addr = smem_u32(sK);
            for (; w.valid(); w.next()) {
                if (w.qb != prev_qb) {
                    const BlockInfo blk = a.blocks[w.qb];
                    const BatchInfo bi = a.batches[blk.b];
                    int nrows = bi.Sq - blk.i0;
                    nrows = nrows > NQ ? NQ : nrows;
                    int n = ((nrows * N1P + 15) / 16) * 16;
                    n = n < 16 ? 16 : (n > kAccCols ? kAccCols : n);
                    idesc = a.idesc_base | ((uint32_t)(n >> 3) << 17);
                    if (!mbar_wait_bounded(q_full, qphase, abort_flag, a.timeout_ns)) {
                        fail(a.hdr, abort_flag, LI_DEV_TIMEOUT);
                        break;
                    }
                    qphase ^= 1u;
                    prev_qb = w.qb;
                }
                if (!mbar_wait_bounded(&k_full[stage], phase, abort_flag, a.timeout_ns) ||
                    !mbar_wait_bounded(&acc_empty[acc], acc_phase ^ 1u, abort_flag, a.timeout_ns)) {
                    fail(a.hdr, abort_flag, LI_DEV_TIMEOUT);
                    break;
                }
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * kAccCols);
                const uint32_t k_addr = sK_addr + stage * G::K_BYTES;
#pragma unroll
                for (int c = 0; c < CHUNKS; ++c) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t ad = smem_desc_sw128(k_addr + c * G::K_CHUNK + kk * 32);
                        const uint64_t bd = smem_desc_sw128(sQ_addr + c * G::Q_CHUNK + kk * 32);
                        if constexpr (KIND == kKindE4M3)
                            mma_f8(d_tmem, ad, bd, idesc, (c | kk) != 0);
                        else if constexpr (KIND == kKindI8)
                            mma_i8(d_tmem, ad, bd, idesc, (c | kk) != 0);
                        else
                            mma_f16(d_tmem, ad, bd, idesc, (c | kk) != 0);
                    }
                }
                issued = true;
                mma_commit(&k_empty[stage]);
                mma_commit(&acc_full[acc]);
                if (w.tile + 1 == w.ntiles) mma_commit(q_empty);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
                if (++acc == kAccStages) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
            if (issued) {
                // every MMA of this CTA has finished before TMEM is released
                mma_commit(drain);
                mbar_wait_bounded(drain, 0, nullptr, a.timeout_ns);
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        // Two groups of eight warps, one per accumulator: group g takes the
        // tiles of accumulator g (every other tile), so one group reduces a
        // tile while the other loads the next, and each has two MMA times
        // per tile.  In a group, each thread owns key row `lrow` of the tile
        // and the 128 columns of its warp half (QPW queries x N1P heads); it
        // streams them out of TMEM 16 at a time, hands the accumulator back
        // once the last chunk is in registers, and reduces
        // sum_h W*ReLU(logit) with packed fp32 FMAs.
        const int ew = warp - 2;                   // 0..15
        const int grp = ew / kGroupWarps;          // the accumulator (tile parity) of this group
        const int quarter = warp & 3;              // TMEM lane quarter this warp may access
        const int half = (ew % kGroupWarps) >> 2;  // which 128 of the 256 columns
        const int lrow = quarter * 32 + lane;      // key row within the tile
        float *myW = sW + ew * 128;
        if (w_begin < w_end && nblocks > 0) {
            Walker w{a.blocks, nblocks, 0, a.q_cost, 0, 0, 0, 0};
            w.init_from(a.cta_start[blockIdx.x], w_end);
            const int acc = grp;
            int prev_qb = -1, nchunks = 0, parity = 0;
            uint32_t acc_phase = 0;
            BlockInfo blk{};
            BatchInfo bi{};
            float *row_ptr = nullptr;              // score row of this half's first query
            int64_t lim0 = 0;                      // visible keys of query q: (lim0 + q) >> cmp_shift
            int nq_valid = 0;                      // valid queries of this warp
            for (; w.valid(); w.next(), parity ^= 1) {
                if (parity != grp) continue;       // the other group's tile
                if (w.qb != prev_qb) {
                    blk = a.blocks[w.qb];
                    bi = a.batches[blk.b];
                    int nrows = bi.Sq - blk.i0;
                    nrows = nrows > NQ ? NQ : nrows;
                    int mine = nrows - half * QPW;     // valid queries of this half
                    mine = mine < 0 ? 0 : (mine > QPW ? QPW : mine);
                    nq_valid = mine;
                    nchunks = (mine * N1P + 15) / 16;   // 16-column chunks
                    const int i_first = blk.i0 + half * QPW;
                    row_ptr = a.scores + (int64_t)(bi.row0 + i_first) * a.ld;
                    // right-down causal over compressed keys (see causal_visible);
                    // mode 0 sees all Sk keys
                    lim0 = a.mode == 3
                               ? (int64_t)i_first + 1 - bi.Sq + ((int64_t)bi.Sk << a.cmp_shift) + bi.res
                               : ((int64_t)bi.Sk << a.cmp_shift);
                    __syncwarp();
                    for (int j = lane; j < 128; j += 32) {
                        const int col = half * 128 + j;
                        const int q = col / N1P, h = col % N1P;
                        const int i = blk.i0 + q;
                        float wv = 0.f;
                        if (h < a.N1 && i < bi.Sq) {
                            const int64_t r = (int64_t)(bi.q_off + i) * a.N1 + h;
                            wv = load_weight(a.weights, a.dtype_w, r);
                            if (a.quant) {
                                const float sq = load_scale(a.q_scale, a.dtype_scale, r);
                                if (sq < 0.f) atomicOr(&a.hdr->status, LI_DEV_NEG_SCALE);
                                wv *= sq;
                            }
                        }
                        myW[j] = fadd_col(j) ? 0.5f * wv : wv;
                    }
                    __syncwarp();
                    prev_qb = w.qb;
                }
                if (!mbar_wait_bounded(&acc_full[acc], acc_phase, abort_flag, a.timeout_ns)) {
                    fail(a.hdr, abort_flag, LI_DEV_TIMEOUT);
                    break;
                }
                tc_fence_after_sync();
                const uint32_t trow = tmem_base + ((uint32_t)(quarter * 32) << 16) +
                                      (uint32_t)(acc * kAccCols + half * 128);
                const int t = w.tile * kTileKeys + lrow;
                float ks = 1.f;
                if (a.quant && t < bi.Sk) {
                    int64_t kr = -1;
                    if (!a.is_pa) {
                        kr = (int64_t)bi.k_off + t;
                    } else {
                        const int id = a.block_table[(int64_t)blk.b * a.max_blocks_per_seq +
                                                     t / a.block_size];
                        if (id >= 0 && id < a.num_blocks)
                            kr = (int64_t)id * a.block_size + t % a.block_size;
                    }
                    if (kr >= 0) {
                        ks = load_scale(a.k_scale, a.dtype_scale, kr);
                        if (ks < 0.f) atomicOr(&a.hdr->status, LI_DEV_NEG_SCALE);
                    }
                }
                uint64_t part[QPW][NP2];
#pragma unroll
                for (int q = 0; q < QPW; ++q)
#pragma unroll
                    for (int p = 0; p < NP2; ++p) part[q][p] = 0ull;
                if (nchunks == 8)
                    epi_reduce<QPW, NP2, N1P, KIND>(trow, 8, myW, part, &acc_empty[acc], lane);
                else if (nchunks > 0)
                    epi_reduce<QPW, NP2, N1P, KIND>(trow, nchunks, myW, part, &acc_empty[acc], lane);
                if (nchunks == 0) {                // nothing to read: release at once
                    tc_fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&acc_empty[acc]);
                }
                acc_phase ^= 1u;
                // visible keys only: t < nvis(i); the row keeps its visible prefix
#pragma unroll
                for (int q = 0; q < QPW; ++q) {
                    if (q < nq_valid) {
                        const int64_t v = (lim0 + q) >> a.cmp_shift;
                        const int nv = v < 0 ? 0 : (v < bi.Sk ? (int)v : bi.Sk);
                        if (t < nv) {
                            float s = 0.f;
#pragma unroll
                            for (int p = 0; p < NP2; ++p) s += hsum2(part[q][p]);
                            row_ptr[(int64_t)q * a.ld + t] = s * ks;
                        }
                    }
                }
            }
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 1) tmem_dealloc(tmem_base, 2 * kAccCols);
}

template <int CHUNKS, int N1P, int KIND>
cudaError_t launch_one(const ScoreArgs &a, const CUtensorMap &qmap, const CUtensorMap &kmap,
                       int grid, cudaStream_t s)
{
    auto kern = score_kernel<CHUNKS, N1P, KIND>;
    const size_t smem = Geometry<CHUNKS>::SMEM;
    cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void *>(kern), (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kScoreThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, qmap, kmap, a);
}

template <int CHUNKS, int KIND>
cudaError_t launch_n1p(const ScoreArgs &a, int n1p, const CUtensorMap &qmap,
                       const CUtensorMap &kmap, int grid, cudaStream_t s)
{
    switch (n1p) {
    case 8: return launch_one<CHUNKS, 8, KIND>(a, qmap, kmap, grid, s);
    case 16: return launch_one<CHUNKS, 16, KIND>(a, qmap, kmap, grid, s);
    case 32: return launch_one<CHUNKS, 32, KIND>(a, qmap, kmap, grid, s);
    case 64: return launch_one<CHUNKS, 64, KIND>(a, qmap, kmap, grid, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

size_t score_smem_bytes(int chunks) { return chunks == 2 ? Geometry<2>::SMEM : Geometry<1>::SMEM; }
int score_stages(int chunks) { return chunks == 2 ? Geometry<2>::STAGES : Geometry<1>::STAGES; }

cudaError_t launch_score(const ScoreArgs &a, const Tiling &t, const CUtensorMap &qmap,
                         const CUtensorMap &kmap, int kind, int grid, cudaStream_t s)
{
    if (kind == kKindE4M3)
        return t.chunks == 1 ? launch_n1p<1, kKindE4M3>(a, t.n1p, qmap, kmap, grid, s) : cudaErrorInvalidValue;
    if (kind == kKindI8)
        return t.chunks == 1 ? launch_n1p<1, kKindI8>(a, t.n1p, qmap, kmap, grid, s) : cudaErrorInvalidValue;
    return t.chunks == 2 ? launch_n1p<2, kKindF16>(a, t.n1p, qmap, kmap, grid, s)
                         : launch_n1p<1, kKindF16>(a, t.n1p, qmap, kmap, grid, s);
}

}  // namespace li
