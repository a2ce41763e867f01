// li_plan.cu -- the device-side scheduler.
//
// The analog of the lightning_indexer_metadata pre-op of the CANN guide
// ("接口分工": a task list giving each core its start/end batch, head and
// Q/K block): it runs on the device, reads the actual lengths where they
// live, and writes a flat list of work units so that the score kernel can
// split the visible (query block, key tile) pairs evenly over all SMs without
// a host synchronisation.
//
// Output (in the workspace):
//   BatchInfo[b]  clamped lengths and offsets of every batch
//   BlockInfo[g]  query block g: its batch, first query, the number of key
//                 tiles its last (most-seeing) query needs, and its first
//                 position in the weighted work list (tiles + q_cost per block)
//   cta_start[c]  where score CTA c's equal share of the work list begins:
//                 its first block, tile, and that block's unit_start and
//                 tile count (one load for the CTA instead of a search)
//   PlanHeader    totals and the device status word (cleared here: this is
//                 the first kernel of every call)
// Lengths outside what the tensors or the declared bounds can hold are
// clamped and reported through LI_DEV_BAD_QLEN / LI_DEV_BAD_KLEN.
#include <cstdint>

#include "li_internal.cuh"
#include "ptx.cuh"

namespace li {
namespace {

__device__ __forceinline__ int64_t clamp64(int64_t v, int64_t lo, int64_t hi)
{
    return v < lo ? lo : (v > hi ? hi : v);
}

// Inclusive scan over the CTA (kPlanThreads threads); returns the total.
__device__ int32_t block_inclusive_scan(int32_t &v, int32_t *tmp)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int W = kPlanThreads / 32;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int32_t y = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += y;
    }
    if (lane == 31) tmp[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int32_t w = lane < W ? tmp[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int32_t y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        if (lane < W) tmp[lane] = w;
    }
    __syncthreads();
    if (warp > 0) v += tmp[warp - 1];
    const int32_t total = tmp[W - 1];
    __syncthreads();
    return total;
}

constexpr int kSmemBatches = 768;       // batches mirrored in shared memory
constexpr int kSmemBlocks = 8192;       // query blocks whose first unit is mirrored

__global__ void __launch_bounds__(kPlanThreads) plan_kernel(PlanArgs a)
{
    __shared__ int32_t s_tmp[kPlanThreads / 32];
    __shared__ int32_t s_flags;
    __shared__ int4 s_bat[kSmemBatches];          // (blk_off, Sq, Sk, res)
    __shared__ int32_t s_ustart[kSmemBlocks];     // unit_start of block g
    const bool in_smem = a.B <= kSmemBatches;
    const int tid = threadIdx.x;
    // let the score kernel's CTAs launch and run their prologue now; its
    // griddepcontrol.wait still waits for this grid's completion and writes
    grid_launch_dependents();
    if (tid == 0) s_flags = 0;
    __syncthreads();

    // 1. per-batch lengths, clamped, and the number of query blocks of each
    int32_t carry = 0;
    for (int base = 0; base < a.B; base += kPlanThreads) {
        const int b = base + tid;
        int32_t nblk = 0;
        int flags = 0;
        BatchInfo bi = {};
        if (b < a.B) {
            int64_t q_off, Sq, k_off, Sk;
            if (a.layout_q == LI_TND) {              // prefix sums, no leading 0
                const int64_t lo = b ? a.act_q[b - 1] : 0, hi = a.act_q[b];
                const int64_t clo = clamp64(lo, 0, a.T1), chi = clamp64(hi, clo, a.T1);
                if (clo != lo || chi != hi) flags |= LI_DEV_BAD_QLEN;
                q_off = clo;
                Sq = chi - clo;
            } else {
                const int64_t s = a.act_q ? a.act_q[b] : a.S1;
                Sq = clamp64(s, 0, a.S1);
                if (Sq != s) flags |= LI_DEV_BAD_QLEN;
                q_off = (int64_t)b * a.S1;
            }
            if (a.layout_k == LI_TND) {
                const int64_t lo = b ? a.act_k[b - 1] : 0, hi = a.act_k[b];
                const int64_t clo = clamp64(lo, 0, a.T2), chi = clamp64(hi, clo, a.T2);
                if (clo != lo || chi != hi) flags |= LI_DEV_BAD_KLEN;
                k_off = clo;
                Sk = chi - clo;
            } else if (a.layout_k == LI_BSND) {
                const int64_t s = a.act_k ? a.act_k[b] : a.S2;
                Sk = clamp64(s, 0, a.S2);
                if (Sk != s) flags |= LI_DEV_BAD_KLEN;
                k_off = (int64_t)b * a.S2;
            } else {                                  // PA: a count per batch
                const int64_t s = a.act_k[b];
                Sk = clamp64(s, 0, a.pa_capacity);
                if (Sk != s) flags |= LI_DEV_BAD_KLEN;
                k_off = 0;
            }
            if (Sk > a.ld) {                          // beyond the declared bound
                Sk = a.ld;
                flags |= LI_DEV_BAD_KLEN;
            }
            bi.q_off = (int32_t)q_off;
            bi.Sq = (int32_t)Sq;
            bi.k_off = (int32_t)k_off;
            bi.Sk = (int32_t)Sk;
            bi.row0 = (int32_t)q_off;
            nblk = (int32_t)((Sq + a.nq - 1) / a.nq);
            bi.nblk = nblk;
            if (a.cmp_res && a.mode == 3) {           // residual tokens: below cmp_ratio
                const int32_t r = a.cmp_res[b], rmax = (1 << a.cmp_shift) - 1;
                bi.res = r < 0 ? 0 : (r > rmax ? rmax : r);
                if (bi.res != r) flags |= LI_DEV_BAD_KLEN;
            }
        }
        if (flags) atomicOr(&s_flags, flags);
        int32_t incl = nblk;
        const int32_t tot = block_inclusive_scan(incl, s_tmp);
        if (b < a.B) {
            bi.blk_off = carry + incl - nblk;
            a.batches[b] = bi;
            if (in_smem) {
                s_bat[b] = make_int4(bi.blk_off, bi.Sq, bi.Sk, bi.res);
            }
        }
        carry += tot;
    }
    int32_t total_blocks = carry;
    if (total_blocks > a.max_blocks) {               // cannot happen for valid params
        total_blocks = a.max_blocks;
        if (tid == 0) atomicOr(&s_flags, LI_DEV_BAD_QLEN);
    }
    __syncthreads();   // batches[] visible to the whole CTA (global writes, same CTA)
    __threadfence_block();

    // 2. every query block: its batch, first query and visible key tiles; the
    //    exclusive scan of the tile counts gives each block's first unit
    carry = 0;
    for (int base = 0; base < total_blocks; base += kPlanThreads) {
        const int g = base + tid;
        int32_t ntiles = 0;
        BlockInfo blk = {};
        if (g < total_blocks) {
            int lo = 0, hi = a.B - 1;                  // last batch with blk_off <= g
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                const int off = in_smem ? s_bat[mid].x : a.batches[mid].blk_off;
                if (off <= g) lo = mid; else hi = mid - 1;
            }
            int32_t blk_off, Sq, Sk, res;
            if (in_smem) {
                const int4 sb = s_bat[lo];
                blk_off = sb.x;
                Sq = sb.y;
                Sk = sb.z;
                res = sb.w;
            } else {
                const BatchInfo bi = a.batches[lo];
                blk_off = bi.blk_off;
                Sq = bi.Sq;
                Sk = bi.Sk;
                res = bi.res;
            }
            const int32_t i0 = (g - blk_off) * a.nq;
            int32_t i_last = i0 + a.nq;
            if (i_last > Sq) i_last = Sq;
            i_last -= 1;
            int64_t nvis = Sk;
            if (a.mode == 3) nvis = causal_visible(i_last, Sq, Sk, res, a.cmp_shift);
            ntiles = (int32_t)((nvis + kTileKeys - 1) / kTileKeys);
            blk.b = lo;
            blk.i0 = i0;
            blk.ntiles = ntiles;
        }
        // a block weighs its key tiles plus the cost of loading its query tile
        const int32_t weight = ntiles > 0 ? ntiles + a.q_cost : 0;
        int32_t incl = weight;
        const int32_t tot = block_inclusive_scan(incl, s_tmp);
        if (g < total_blocks) {
            blk.unit_start = carry + incl - weight;
            a.blocks[g] = blk;
            if (g < kSmemBlocks) s_ustart[g] = blk.unit_start;
        }
        carry += tot;
    }

    // 3. the start of every score CTA's share [total*c/grid, total*(c+1)/grid)
    //    of the work list: the last block whose first unit is at or before
    //    the share's first unit w0, and the tile of w0 inside it.  Blocks
    //    without tiles share their first unit with the next block, so the
    //    last such block always has the tile (w0 < its end, or the next block
    //    would start at or before w0).
    const int32_t total_units = carry;
    __syncthreads();   // s_ustart and blocks[] visible to the whole CTA
    const bool ustart_in_smem = total_blocks <= kSmemBlocks;
    for (int c = tid; c < a.grid; c += kPlanThreads) {
        int4 st = make_int4(0, 0, 0, 0);
        if (total_blocks > 0 && total_units > 0) {
            const int32_t w0 = (int32_t)(((int64_t)total_units * c) / a.grid);
            int lo = 0, hi = total_blocks - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                const int32_t u = ustart_in_smem ? s_ustart[mid] : a.blocks[mid].unit_start;
                if (u <= w0) lo = mid; else hi = mid - 1;
            }
            const int32_t u0 = ustart_in_smem ? s_ustart[lo] : a.blocks[lo].unit_start;
            const int32_t u1 = lo + 1 < total_blocks
                                   ? (ustart_in_smem ? s_ustart[lo + 1] : a.blocks[lo + 1].unit_start)
                                   : total_units;
            int32_t tile = w0 - u0 - a.q_cost;
            if (tile < 0) tile = 0;
            st = make_int4(lo, tile, u0, u1 - u0 - a.q_cost);
        }
        a.cta_start[c] = st;
    }
    if (tid == 0) {
        a.hdr->total_blocks = total_blocks;
        a.hdr->total_units = carry;
        a.hdr->status = s_flags;
    }
}

// Bounded-wait self test: wait on a barrier that nothing completes.
__global__ void wait_selftest_kernel(int32_t *status, int64_t timeout_ns)
{
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        abort_flag = 0;
        mbar_init(&bar, 1);
        fence_mbarrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        if (!mbar_wait_bounded(&bar, 0, &abort_flag, timeout_ns))
            atomicOr(status, LI_DEV_TIMEOUT);
    }
    __syncthreads();
}

}  // namespace

cudaError_t launch_plan(const PlanArgs &a, cudaStream_t s)
{
    plan_kernel<<<1, kPlanThreads, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_wait_selftest(int32_t *status, int64_t timeout_ns, cudaStream_t s)
{
    wait_selftest_kernel<<<1, 32, 0, s>>>(status, timeout_ns);
    return cudaGetLastError();
}

}  // namespace li
