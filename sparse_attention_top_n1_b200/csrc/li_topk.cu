// li_topk.cu -- per-row Top-k over fp32 score rows.
//
// Step 3 of the CANN LightningIndexerV2 guide ("三步计算流程": keep the k
// best positions) with the deterministic order of its "确定性计算" section,
// read as: value descending, ties by lower key index; slots past the number
// of candidates hold -1 / -inf ("通用约束").
//
// Rows of up to 16384 keys: one CTA of 512 threads per row.
//   The row is cached in shared memory as order-preserving uint32 keys
//   (-0.0 folded into +0.0).  The bucket path histograms it over 2048 linear
//   value buckets between its min and max, finds the bucket holding the k-th
//   largest value, scatters the selected keys grouped by bucket, and gives
//   each its final slot: its bucket's offset plus its rank inside the bucket,
//   counted by (value desc, index asc).  When a bucket is too full for
//   counting (ties, clustered values) or the range is degenerate, the exact
//   radix path runs instead:
//   1. Radix select: three histogram passes (11, 11 and 10 bits, most
//      significant first) find the exact key T of the k-th largest element
//      and how many of the k come from the elements equal to T.
//   2. Compaction in index order: every key > T, plus the lowest-index keys
//      == T.
//   3. A stable LSB radix sort by descending value (4 passes of 8 bits; a
//      pass whose digit is the same for every selected key is skipped).
//   4. Write indices and values, pad with -1 / -inf.
// Longer rows (decode over long contexts): a thread-block cluster of 8 CTAs
// per row runs the bucket method over distributed shared memory (see the
// long-rows section below).
#include <cstdint>
#include <cooperative_groups.h>

#include "li_internal.cuh"
#include "ptx.cuh"

namespace li {
namespace {

constexpr int kMaxWarps = 16;        // CTAs have at most 512 threads

__device__ __forceinline__ uint32_t to_key(float f)
{
    f = f + 0.0f;                                  // -0.0 -> +0.0
    uint32_t b = __float_as_uint(f);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ float from_key(uint32_t u)
{
    uint32_t b = (u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u;
    return __uint_as_float(b);
}

__device__ __forceinline__ uint32_t lanemask_lt()
{
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Exclusive scan of one value per thread over the whole CTA of NT threads;
// also returns the total.  `tmp` holds NT/32 + 1 values.  Contains __syncthreads.
template <int NT, typename T>
__device__ __forceinline__ T block_exclusive_scan(T v, T *tmp, T &total)
{
    constexpr int kWarps = NT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    T x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        T y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) tmp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        T w = lane < kWarps ? tmp[lane] : T(0);
        T s = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            T y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        if (lane < kWarps) tmp[lane] = s - w;          // exclusive warp offsets
        if (lane == kWarps - 1) tmp[kWarps] = s;       // total
    }
    __syncthreads();
    T r = tmp[warp] + x - v;
    total = tmp[kWarps];
    __syncthreads();
    return r;
}

__device__ __forceinline__ uint32_t warp_min(uint32_t v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ uint32_t warp_max(uint32_t v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ uint32_t warp_or(uint32_t v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v |= __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ uint32_t warp_and(uint32_t v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v &= __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

struct RowSrc {
    const float *g;       // row in global memory
    const uint32_t *c;    // row cached as keys in shared memory (or null)
    int n;
    __device__ __forceinline__ uint4 load4(int j4) const
    {
        // keys j4*4 .. j4*4+3; entries >= n are never used by callers
        if (c) return reinterpret_cast<const uint4 *>(c)[j4];
        float4 v = reinterpret_cast<const float4 *>(g)[j4];
        return make_uint4(to_key(v.x), to_key(v.y), to_key(v.z), to_key(v.w));
    }
};

struct TopkSmem {
    uint32_t *hist;     // 4096 words: radix histograms, or bucket counts + cursors
    uint32_t *keyA;     // kmax selected keys
    int32_t *idxA;
    uint32_t *candK;    // threshold-bucket candidates of the bucket path
    int32_t *candI;
    uint32_t *keyB;     // kmax: radix ping-pong buffer (aliases the cache, dead by then)
    int32_t *idxB;
    uint32_t *cache;    // the row as keys, when it fits
};

constexpr int kMaxCluster = 8;       // CTAs per row for the longest rows

struct TopkShared {
    uint32_t tmp32[kMaxWarps + 1];
    uint64_t tmp64[kMaxWarps + 1];
    uint32_t digit, above, vor, vand, kmin, kmax, maxbin;
    uint32_t pmin[kMaxCluster], pmax[kMaxCluster];   // slice ranges pushed by the cluster
    uint32_t verdict;                                // CTA 0 -> all: bucket method taken
    uint32_t bstar, above_b;                         // CTA 0 -> all: threshold bucket
};

// ---------------------------------------------------------------- radix path
// Exact for every input (ties, equal values, any range): three histogram
// passes find the k-th key, an index-order compaction selects, a stable LSB
// radix sort orders.  Used when the bucket path declines a row.
// Keys j < fa and j >= fc are forced (sink tokens and local window): they
// take part in the selection as the largest possible key and are ordered by
// their real key (fa = 0, fc = n: none forced).
template <int NT, int KMAX>
__device__ void radix_topk(const RowSrc &src, int n, int k, int m, const TopkSmem &s,
                           TopkShared &sh, int32_t *oidx, float *oval, int fa, int fc)
{
    constexpr int kTopkThreads = NT, kWarps = NT / 32;
    constexpr int kSortMaxRounds = KMAX / NT;       // rounds of 32 per warp for kmax <= KMAX
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n4 = (n + 3) >> 2;
    uint32_t *hist = s.hist, *keyA = s.keyA, *keyB = s.keyB;
    int32_t *idxA = s.idxA, *idxB = s.idxB;
    uint32_t *s_tmp32 = sh.tmp32;
    uint64_t *s_tmp64 = sh.tmp64;
    uint32_t &s_digit = sh.digit, &s_above = sh.above, &s_or = sh.vor, &s_and = sh.vand;
    // radix select of the k-th largest key (only when n > k)
    uint32_t T = 0;
    int need_eq = 0;
    if (n > k) {
        uint32_t prefix = 0, pmask = 0;
        int remaining = k;
        const int shifts[3] = {21, 10, 0};
        const int widths[3] = {11, 11, 10};
#pragma unroll
        for (int pass = 0; pass < 3; ++pass) {
            const int shift = shifts[pass], bins = 1 << widths[pass];
            const uint32_t dmask = (uint32_t)bins - 1u;
            for (int j = tid; j < bins; j += kTopkThreads) hist[j] = 0;
            __syncthreads();
            // every lane runs the same number of iterations (match_any below)
            for (int base4 = 0; base4 < n4; base4 += kTopkThreads) {
                const int j4 = base4 + tid;
                uint32_t kv[4] = {0, 0, 0, 0};
                if (j4 < n4) {
                    uint4 q = src.load4(j4);
                    kv[0] = q.x; kv[1] = q.y; kv[2] = q.z; kv[3] = q.w;
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = j4 * 4 + e;
                    const uint32_t sk = (j < fa || j >= fc) ? 0xFFFFFFFFu : kv[e];   // selection key
                    const bool act = j < n && (sk & pmask) == prefix;
                    const uint32_t d = act ? (sk >> shift) & dmask : 0xFFFFFFFFu;
                    const uint32_t peers = __match_any_sync(0xffffffffu, d);
                    if (act && (peers & lanemask_lt()) == 0)
                        atomicAdd(&hist[d], (uint32_t)__popc(peers));
                }
            }
            __syncthreads();
            // thread t owns `per` consecutive bins, counted from the top digit down
            const int per = bins / kTopkThreads;
            uint32_t c = 0;
            for (int e = 0; e < per; ++e) c += hist[bins - 1 - (tid * per + e)];
            uint32_t tot;
            uint32_t above = block_exclusive_scan<NT, uint32_t>(c, s_tmp32, tot);
            if (above < (uint32_t)remaining && above + c >= (uint32_t)remaining) {
                uint32_t acc = above;
                for (int e = 0; e < per; ++e) {
                    const int d = bins - 1 - (tid * per + e);
                    const uint32_t h = hist[d];
                    if (acc + h >= (uint32_t)remaining) {
                        s_digit = (uint32_t)d;
                        s_above = acc;
                        break;
                    }
                    acc += h;
                }
            }
            __syncthreads();
            remaining -= (int)s_above;
            prefix |= s_digit << shift;
            pmask |= dmask << shift;
            __syncthreads();
        }
        T = prefix;
        need_eq = remaining;
    }

    // --- 2. compaction in index order into keyA/idxA
    if (n <= k) {
        for (int j4 = tid; j4 < n4; j4 += kTopkThreads) {
            uint4 q = src.load4(j4);
            uint32_t kv[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int j = j4 * 4 + e;
                if (j < n) { keyA[j] = kv[e]; idxA[j] = j; }
            }
        }
    } else {
        uint32_t gt_carry = 0, eq_carry = 0;
        for (int base4 = 0; base4 < n4; base4 += kTopkThreads) {
            const int j4 = base4 + tid;
            uint32_t kv[4] = {0, 0, 0, 0};
            uint32_t ngt = 0, neq = 0;
            if (j4 < n4) {
                uint4 q = src.load4(j4);
                kv[0] = q.x; kv[1] = q.y; kv[2] = q.z; kv[3] = q.w;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = j4 * 4 + e;
                    const uint32_t sk = (j < fa || j >= fc) ? 0xFFFFFFFFu : kv[e];
                    if (j < n) { ngt += sk > T; neq += sk == T; }
                }
            }
            uint64_t packed = ((uint64_t)neq << 32) | ngt, tot;
            uint64_t before = block_exclusive_scan<NT, uint64_t>(packed, s_tmp64, tot);
            uint32_t gt_b = gt_carry + (uint32_t)before;
            uint32_t eq_b = eq_carry + (uint32_t)(before >> 32);
            if (j4 < n4) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = j4 * 4 + e;
                    if (j >= n) break;
                    const uint32_t sk = (j < fa || j >= fc) ? 0xFFFFFFFFu : kv[e];
                    const bool gt = sk > T, eq = sk == T;
                    if (gt || (eq && eq_b < (uint32_t)need_eq)) {
                        const uint32_t pos = gt_b + (eq_b < (uint32_t)need_eq ? eq_b : (uint32_t)need_eq);
                        keyA[pos] = kv[e];
                        idxA[pos] = j;
                    }
                    gt_b += gt;
                    eq_b += eq;
                }
            }
            gt_carry += (uint32_t)tot;
            eq_carry += (uint32_t)(tot >> 32);
        }
    }
    __syncthreads();

    // --- 3. stable LSB radix sort of keyA/idxA (m elements) by descending key
    uint32_t *kin = keyA, *kout = keyB;
    int32_t *iin = idxA, *iout = idxB;
    if (m > 1) {
        if (tid == 0) { s_or = 0; s_and = 0xFFFFFFFFu; }
        __syncthreads();
        uint32_t vor = 0, vand = 0xFFFFFFFFu;
        for (int j = tid; j < m; j += kTopkThreads) { vor |= kin[j]; vand &= kin[j]; }
        vor = warp_or(vor);
        vand = warp_and(vand);
        if (lane == 0) {                    // one shared atomic per warp, not per thread
            atomicOr(&s_or, vor);
            atomicAnd(&s_and, vand);
        }
        __syncthreads();
        const uint32_t diff = s_or ^ s_and;
        const int seg = (((m + kWarps - 1) / kWarps) + 31) & ~31;     // elements per warp
        const int rounds = seg >> 5;
        uint32_t *whist = hist + warp * 256;                            // per-warp digit counts
        for (int shift = 0; shift < 32; shift += 8) {
            if (((diff >> shift) & 0xFFu) == 0) continue;               // same digit everywhere
            for (int j = lane; j < 256; j += 32) whist[j] = 0;
            __syncwarp();
            uint32_t local[kSortMaxRounds];
            const int wbeg = warp * seg;
#pragma unroll
            for (int r = 0; r < kSortMaxRounds; ++r) {
                if (r >= rounds) break;
                const int e = wbeg + r * 32 + lane;
                const bool valid = e < m;
                const uint32_t d = valid ? ((~kin[e]) >> shift) & 0xFFu : 0xFFFFFFFFu;
                const uint32_t peers = __match_any_sync(0xffffffffu, d);
                uint32_t cnt = 0;
                if (valid) cnt = whist[d];
                local[r] = cnt + __popc(peers & lanemask_lt());
                __syncwarp();
                if (valid && (peers & lanemask_lt()) == 0) whist[d] = cnt + __popc(peers);
                __syncwarp();
            }
            __syncthreads();
            // exclusive scan over (digit major, warp minor): thread t owns the
            // 8 consecutive counters 8t .. 8t+7 of that order
            uint32_t own[8], sum = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int c = tid * 8 + j, d = c / kWarps, wi = c % kWarps;
                own[j] = hist[wi * 256 + d];
                sum += own[j];
            }
            uint32_t tot;
            uint32_t off = block_exclusive_scan<NT, uint32_t>(sum, s_tmp32, tot);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int c = tid * 8 + j, d = c / kWarps, wi = c % kWarps;
                hist[wi * 256 + d] = off;
                off += own[j];
            }
            __syncthreads();
#pragma unroll
            for (int r = 0; r < kSortMaxRounds; ++r) {
                if (r >= rounds) break;
                const int e = wbeg + r * 32 + lane;
                if (e < m) {
                    const uint32_t kk = kin[e];
                    const uint32_t d = ((~kk) >> shift) & 0xFFu;
                    const uint32_t dst = whist[d] + local[r];
                    kout[dst] = kk;
                    iout[dst] = iin[e];
                }
            }
            __syncthreads();
            uint32_t *tk = kin; kin = kout; kout = tk;
            int32_t *ti = iin; iin = iout; iout = ti;
        }
    }

    // write out
    for (int j = tid; j < k; j += kTopkThreads) {
        if (j < m) {
            oidx[j] = iin[j];
            if (oval) oval[j] = from_key(kin[j]);
        } else {
            oidx[j] = -1;
            if (oval) oval[j] = __uint_as_float(0xFF800000u);
        }
    }
}

// ---------------------------------------------------------------- bucket path
// Linear value buckets over [min, max] of the row (monotone in the value):
// one histogram pass finds the bucket holding the m-th largest value, one
// scatter pass groups the selected elements by bucket, and each element's
// final rank is its bucket's offset plus its rank inside the bucket, counted
// by comparing (value desc, index asc) with the bucket's other members.
// Declines (returns false, uniformly, before writing anything) when a
// bucket is too full for counting to be cheap or the range is degenerate.
constexpr int kBuckets = 2048;
constexpr int kBinLimit = 64;       // largest selected bucket ranked by counting
constexpr int kCandLimit = 512;     // largest threshold bucket resolved by counting

__device__ __forceinline__ int bucket_of(uint32_t key, float fmin, float scale)
{
    const int b = __float2int_rz((from_key(key) - fmin) * scale);
    return b < 0 ? 0 : (b >= kBuckets ? kBuckets - 1 : b);
}

__device__ bool bucket_topk(const RowSrc &src, int n, int k, int m, int kmax, const TopkSmem &s,
                            TopkShared &sh, int32_t *oidx, float *oval)
{
    const int tid = threadIdx.x;
    const float fmin = from_key(sh.kmin), fmax = from_key(sh.kmax);
    const float range = fmax - fmin;
    if (!(range > 0.f) || !isfinite(range)) return false;
    const float scale = (float)kBuckets / range;
    if (!isfinite(scale)) return false;
    uint32_t *hist = s.hist, *cur = s.hist + kBuckets;
    const int n4 = (n + 3) >> 2;

    for (int j = tid; j < kBuckets; j += kTopkThreads) hist[j] = 0;
    if (tid == 0) sh.maxbin = 0;
    __syncthreads();
    for (int j4 = tid; j4 < n4; j4 += kTopkThreads) {
        const uint4 q = src.load4(j4);
        const uint32_t kv[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
            if (j4 * 4 + e < n) atomicAdd(&hist[bucket_of(kv[e], fmin, scale)], 1u);
    }
    __syncthreads();

    // buckets from the top down: thread t owns buckets kBuckets-1-(t*per+e)
    constexpr int per = kBuckets / kTopkThreads;
    uint32_t c = 0;
#pragma unroll
    for (int e = 0; e < per; ++e) c += hist[kBuckets - 1 - (tid * per + e)];
    uint32_t tot;
    const uint32_t above_t = block_exclusive_scan<kTopkThreads, uint32_t>(c, sh.tmp32, tot);
    uint32_t acc = above_t;
#pragma unroll
    for (int e = 0; e < per; ++e) {
        const int d = kBuckets - 1 - (tid * per + e);
        const uint32_t h = hist[d];
        if (acc < (uint32_t)m && acc + h >= (uint32_t)m) {
            sh.digit = (uint32_t)d;
            sh.above = acc;
        }
        cur[d] = acc;                       // first slot of bucket d
        acc += h;
    }
    __syncthreads();
    const int bstar = (int)sh.digit;
    const uint32_t above = sh.above;
    const uint32_t cstar = hist[bstar];
    uint32_t lmax = 0;
#pragma unroll
    for (int e = 0; e < per; ++e) {
        const int d = kBuckets - 1 - (tid * per + e);
        if (d > bstar) lmax = max(lmax, hist[d]);
    }
    lmax = warp_max(lmax);
    if ((tid & 31) == 0 && lmax) atomicMax(&sh.maxbin, lmax);
    __syncthreads();
    if (sh.maxbin > (uint32_t)kBinLimit || cstar > (uint32_t)kCandLimit) return false;

    // scatter: selected buckets into their bucket slots, the threshold bucket
    // into the candidate list.  Each key travels as one 64-bit word,
    // (key << 32) | ~index, so that one compare orders by value and, for equal
    // values, by lower index; the words overlay keyA/idxA and candK/candI.
    uint64_t *wA = reinterpret_cast<uint64_t *>(s.keyA);
    uint64_t *wC = reinterpret_cast<uint64_t *>(s.candK);
    for (int j4 = tid; j4 < n4; j4 += kTopkThreads) {
        const uint4 q = src.load4(j4);
        const uint32_t kv[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int j = j4 * 4 + e;
            if (j >= n) break;
            const int b = bucket_of(kv[e], fmin, scale);
            const uint64_t word = ((uint64_t)kv[e] << 32) | (uint32_t)~(uint32_t)j;
            if (b > bstar) {
                const uint32_t pos = atomicAdd(&cur[b], 1u);
                wA[pos] = word;
            } else if (b == bstar) {
                const uint32_t pos = atomicAdd(&cur[b], 1u) - above;
                wC[pos] = word;
            }
        }
    }
    __syncthreads();

    // the threshold bucket: keep the `need` best, ranked among themselves
    const uint32_t need = (uint32_t)m - above;
    for (uint32_t e = tid; e < cstar; e += kTopkThreads) {
        const uint64_t w = wC[e];
        uint32_t r = 0;
        for (uint32_t q = 0; q < cstar; ++q) r += wC[q] > w;
        if (r < need) {
            oidx[above + r] = (int32_t)~(uint32_t)w;
            if (oval) oval[above + r] = from_key((uint32_t)(w >> 32));
        }
    }
    // the buckets above it: bucket offset + rank inside the bucket
    for (uint32_t p = tid; p < above; p += kTopkThreads) {
        const uint64_t w = wA[p];
        const uint32_t kv = (uint32_t)(w >> 32);
        const int b = bucket_of(kv, fmin, scale);
        const uint32_t cnt = hist[b], s0 = cur[b] - cnt;
        uint32_t r = 0;
        for (uint32_t q = s0; q < s0 + cnt; ++q) r += wA[q] > w;
        oidx[s0 + r] = (int32_t)~(uint32_t)w;
        if (oval) oval[s0 + r] = from_key(kv);
    }
    for (int j = m + tid; j < k; j += kTopkThreads) {
        oidx[j] = -1;
        if (oval) oval[j] = __uint_as_float(0xFF800000u);
    }
    return true;
}

template <int KMAX>
__global__ void __launch_bounds__(kTopkThreads) topk_kernel(TopkArgs a)
{
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ TopkShared sh;

    const int tid = threadIdx.x;
    const int row = blockIdx.x;
    const int k = a.k;
    grid_dependency_wait();             // the score rows come from the previous kernel

    // --- which elements of which row
    int n = 0;
    if (a.standalone) {
        n = a.row_len ? a.row_len[row] : (int)a.ld;
        n = n < 0 ? 0 : (n > a.ld ? (int)a.ld : n);
    } else {
        int b = -1, i = 0;
        if (a.layout_q == LI_BSND) {
            b = row / a.S1;
            i = row % a.S1;
        } else {
            int lo = 0, hi = a.B - 1;               // last batch with q_off <= row
            while (lo < hi) {
                int mid = (lo + hi + 1) >> 1;
                if (a.batches[mid].q_off <= row) lo = mid; else hi = mid - 1;
            }
            b = lo;
            i = row - a.batches[b].q_off;
        }
        const BatchInfo bi = a.batches[b];
        if (i >= 0 && i < bi.Sq)
            n = a.mode == 3 ? causal_visible(i, bi.Sq, bi.Sk, bi.res, a.cmp_shift) : bi.Sk;
    }
    int32_t *oidx = a.out_idx + (int64_t)row * k;
    float *oval = a.out_val ? a.out_val + (int64_t)row * k : nullptr;
    const int m = n < k ? n : k;

    if (m == 0) {
        for (int j = tid; j < k; j += kTopkThreads) {
            oidx[j] = -1;
            if (oval) oval[j] = __uint_as_float(0xFF800000u);
        }
        return;
    }

    TopkSmem s;
    s.hist = reinterpret_cast<uint32_t *>(smem);
    s.keyA = s.hist + 4096;
    s.idxA = reinterpret_cast<int32_t *>(s.keyA + a.kmax);
    s.candK = reinterpret_cast<uint32_t *>(s.idxA + a.kmax);
    s.candI = reinterpret_cast<int32_t *>(s.candK + kCandLimit);
    s.cache = reinterpret_cast<uint32_t *>(s.candI + kCandLimit);
    s.keyB = s.cache;                                   // used only after the cache is dead
    s.idxB = reinterpret_cast<int32_t *>(s.cache + a.kmax);

    if (tid == 0) {
        sh.kmin = 0xFFFFFFFFu;
        sh.kmax = 0u;
    }
    __syncthreads();
    RowSrc src;
    src.g = a.scores + (int64_t)row * a.ld;
    src.c = nullptr;
    src.n = n;
    const int n4 = (n + 3) >> 2;
    const bool cached = n <= a.cap;
    uint32_t lmin = 0xFFFFFFFFu, lmax = 0u;
    {
        const float4 *g4 = reinterpret_cast<const float4 *>(src.g);
        uint4 *c4 = reinterpret_cast<uint4 *>(s.cache);
        for (int j4 = tid; j4 < n4; j4 += kTopkThreads) {
            const float4 v = g4[j4];
            const uint4 q = make_uint4(to_key(v.x), to_key(v.y), to_key(v.z), to_key(v.w));
            if (cached) c4[j4] = q;
            const uint32_t kv[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if (j4 * 4 + e < n) {
                    lmin = min(lmin, kv[e]);
                    lmax = max(lmax, kv[e]);
                }
        }
    }
    lmin = warp_min(lmin);
    lmax = warp_max(lmax);
    if ((tid & 31) == 0) {                  // one shared atomic per warp, not per thread
        atomicMin(&sh.kmin, lmin);
        atomicMax(&sh.kmax, lmax);
    }
    if (cached) src.c = s.cache;
    __syncthreads();

    // sink tokens [0, fa) and the local window [fc, n) are always selected
    const int fa = a.init_num < n ? a.init_num : n;
    const int fc = (n - a.local_num) > fa ? n - a.local_num : fa;
    if (fa > 0 || fc < n || !bucket_topk(src, n, k, m, a.kmax, s, sh, oidx, oval))
        radix_topk<kTopkThreads, KMAX>(src, n, k, m, s, sh, oidx, oval, fa, fc);
}

// Number of candidate keys of a row: the visible prefix of the batch's keys
// (indexer mode) or row_len[row] (standalone mode).
__device__ __forceinline__ int row_length(const TopkArgs &a, int row)
{
    if (a.standalone) {
        const int n = a.row_len ? a.row_len[row] : (int)a.ld;
        return n < 0 ? 0 : (n > a.ld ? (int)a.ld : n);
    }
    int b, i;
    if (a.layout_q == LI_BSND) {
        b = row / a.S1;
        i = row % a.S1;
    } else {
        int lo = 0, hi = a.B - 1;                   // last batch with q_off <= row
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (a.batches[mid].q_off <= row) lo = mid; else hi = mid - 1;
        }
        b = lo;
        i = row - a.batches[b].q_off;
    }
    const BatchInfo bi = a.batches[b];
    if (i < 0 || i >= bi.Sq) return 0;
    if (a.mode != 3) return bi.Sk;
    return causal_visible(i, bi.Sq, bi.Sk, bi.res, a.cmp_shift);
}

template <int NT>
__device__ __forceinline__ void pad_row(int32_t *oidx, float *oval, int from, int k)
{
    for (int j = from + (int)threadIdx.x; j < k; j += NT) {
        oidx[j] = -1;
        if (oval) oval[j] = __uint_as_float(0xFF800000u);
    }
}

// Barrier over the whole cluster (C > 1) or the CTA.  A cluster barrier
// orders the shared-memory writes of every CTA before the reads after it.
template <int C>
__device__ __forceinline__ void csync()
{
    if constexpr (C > 1) cooperative_groups::this_cluster().sync();
    else __syncthreads();
}

// The same shared-memory object in CTA `rank` of this cluster.
template <int C, typename T>
__device__ __forceinline__ T *peer(T *p, int rank)
{
    if constexpr (C > 1) return cooperative_groups::this_cluster().map_shared_rank(p, rank);
    else return p;
}

// ---------------------------------------------------------------- long rows
// Rows longer than one CTA caches (decode over long contexts) are split over a
// thread-block cluster of C CTAs, CTA r owning the r-th slice of the row.  The
// bucket method runs cluster-wide through distributed shared memory:
//   1. every CTA pushes its slice's min/max to all CTAs of the cluster;
//   2. every CTA histograms its slice over kCBuckets linear value buckets and
//      adds the counts into CTA 0;
//   3. CTA 0 scans the buckets from the top, finds the bucket holding the
//      m-th largest value and broadcasts it (or declines, as the one-CTA
//      bucket path does);
//   4. every CTA reserves room in CTA 0 bucket by bucket and scatters its
//      selected keys there;
//   5. CTA 0 ranks each key inside its bucket and writes the row.
// A declined row is done by CTA 0 with the exact radix method, streamed.
constexpr int kCBuckets = 2048;      // 52 KB per CTA: the 512 CTAs of 64 long rows fit one wave

// One row per cluster of C CTAs of NT threads; each thread holds up to EPT
// scores of its CTA's slice in registers (float4 group g of thread t covers
// slice keys 4*(t + g*NT) .. +3).  Selected keys travel as one 64-bit word,
// (order-preserving key << 32) | ~index, so that a larger word means a larger
// value or, for equal values, a lower index.
// Four CTAs per SM (registers capped at 32), so the 512 CTAs of 64 long rows
// run as one wave; with k above 2048 the selection buffers allow one CTA per
// SM, and the register cap is lifted.
template <int C, int NT, int EPT, int KMAX>
__global__ void __launch_bounds__(NT, KMAX > 2048 ? 1 : 4) topk_cluster_kernel(TopkArgs a)
{
    constexpr int G = EPT / 4;                  // float4 groups per thread
    constexpr int PER_T = kCBuckets / NT;        // buckets per thread in the scan
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ TopkShared sh;

    const int tid = threadIdx.x;
    int rank = 0;
    if constexpr (C > 1) rank = (int)cooperative_groups::this_cluster().block_rank();
    const int row = blockIdx.x / C;
    const int k = a.k;
    grid_dependency_wait();             // the score rows come from the previous kernel

    const int n = row_length(a, row);
    int32_t *oidx = a.out_idx + (int64_t)row * k;
    float *oval = a.out_val ? a.out_val + (int64_t)row * k : nullptr;
    const int m = n < k ? n : k;
    if (m == 0) {                       // the same in every CTA of the cluster
        if (rank == 0) pad_row<NT>(oidx, oval, 0, k);
        return;
    }

    // shared memory: bucket counts | bucket cursors | selected words | their
    // buckets | tail (candidates + row counts, or the radix sort's buffer)
    uint32_t *hist = reinterpret_cast<uint32_t *>(smem);
    uint32_t *cur = hist + kCBuckets;
    uint64_t *sel = reinterpret_cast<uint64_t *>(cur + kCBuckets);
    uint16_t *selb = reinterpret_cast<uint16_t *>(sel + a.kmax);
    uint32_t *tail = reinterpret_cast<uint32_t *>(selb + a.kmax);
    uint64_t *cand = reinterpret_cast<uint64_t *>(tail);
    uint32_t *gcnt = tail + 2 * kCandLimit;

    const float *grow = a.scores + (int64_t)row * a.ld;
    // sink tokens [0, fa) and the local window [fc, n) are always selected
    const int fa = a.init_num < n ? a.init_num : n;
    const int fc = (n - a.local_num) > fa ? n - a.local_num : fa;
    // whole row with the exact radix method, streamed from global memory (CTA 0)
    auto radix_row = [&]() {
        TopkSmem s;
        s.hist = hist;
        s.keyA = reinterpret_cast<uint32_t *>(sel);
        s.idxA = reinterpret_cast<int32_t *>(s.keyA + a.kmax);
        s.keyB = tail;
        s.idxB = reinterpret_cast<int32_t *>(tail + a.kmax);
        RowSrc full;
        full.g = grow;
        full.c = nullptr;
        full.n = n;
        radix_topk<NT, KMAX>(full, n, k, m, s, sh, oidx, oval, fa, fc);
    };
    if (n > C * NT * EPT || fa > 0 || fc < n) {   // too long, or keys forced in
        if (rank == 0) radix_row();
        return;
    }

    // this CTA's slice [lo, hi) of the row; lo is a multiple of 4
    const int per = (((n + C - 1) / C) + 3) & ~3;
    const int lo = min(n, rank * per), hi = min(n, lo + per);
    const int len = hi - lo;
    const int n4 = (len + 3) >> 2;

    // ---- 1. the slice into registers; push its range to the cluster
    if (tid == 0) {
        sh.kmin = 0xFFFFFFFFu;
        sh.kmax = 0u;
        sh.maxbin = 0u;
    }
    for (int j = tid; j < kCBuckets; j += NT) hist[j] = 0;
    if (C > 1 && rank == 0)
        for (int j = tid; j < kCBuckets; j += NT) gcnt[j] = 0;
    float v[G][4];
    {
        const float4 *g4 = reinterpret_cast<const float4 *>(grow + lo);
        float lmin = __int_as_float(0x7F800000), lmax = __int_as_float(0xFF800000);
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const int j4 = tid + g * NT;
            if (j4 < n4) {
                const float4 x = g4[j4];
                v[g][0] = x.x;
                v[g][1] = x.y;
                v[g][2] = x.z;
                v[g][3] = x.w;
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if (j4 * 4 + e < len) {
                        lmin = fminf(lmin, v[g][e]);
                        lmax = fmaxf(lmax, v[g][e]);
                    }
            }
        }
        // NaN scores are skipped by fminf / fmaxf; their order is unspecified
        uint32_t kmn = to_key(lmin), kmx = to_key(lmax);
        kmn = warp_min(kmn);
        kmx = warp_max(kmx);
        __syncthreads();                // sh initialised
        if ((tid & 31) == 0) {          // one shared atomic per warp, not per thread
            atomicMin(&sh.kmin, kmn);
            atomicMax(&sh.kmax, kmx);
        }
    }
    __syncthreads();
    if (tid < C) {                      // thread r tells CTA r this slice's range
        TopkShared *ps = peer<C>(&sh, tid);
        ps->pmin[rank] = sh.kmin;
        ps->pmax[rank] = sh.kmax;
    }
    csync<C>();                         // S1: ranges pushed, counts cleared

    uint32_t kmin = sh.pmin[0], kmax = sh.pmax[0];
#pragma unroll
    for (int r = 1; r < C; ++r) {
        kmin = min(kmin, sh.pmin[r]);
        kmax = max(kmax, sh.pmax[r]);
    }
    const float fmin = from_key(kmin), fmax = from_key(kmax);
    const float range = fmax - fmin;
    const float scale = (float)kCBuckets / range;
    const float boff = -fmin * scale;
    if (!(range > 0.f) || !isfinite(range) || !isfinite(scale) || !isfinite(boff)) {
        if (rank == 0) radix_row();     // one value, or non-finite scores
        return;
    }
    // bucket of a score: floor(x * scale + boff), clamped; monotone in x
    auto bucket = [&](float x) {
        const int b = __float2int_rz(fmaf(x, scale, boff));
        return b < 0 ? 0 : (b >= kCBuckets ? kCBuckets - 1 : b);
    };

    // ---- 2. histogram of the slice; CTA 0 gathers the row's counts
#pragma unroll
    for (int g = 0; g < G; ++g)
        if (tid + g * NT < n4)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if ((tid + g * NT) * 4 + e < len) atomicAdd(&hist[bucket(v[g][e])], 1u);
    uint32_t *gc = hist;                // the row's counts (one CTA: its own)
    if constexpr (C > 1) {
        __syncthreads();
        uint32_t *g0 = peer<C>(gcnt, 0);
        for (int j = tid; j < kCBuckets; j += NT)
            if (hist[j]) atomicAdd(&g0[j], hist[j]);
        gc = gcnt;                      // meaningful in CTA 0
    }
    csync<C>();                         // S2: CTA 0 holds the row's counts

    // ---- 3. CTA 0: threshold bucket, bucket offsets and the verdict
    if (rank == 0) {
        // thread t owns buckets kCBuckets-1-(t*PER_T+e), counted from the top;
        // a bucket lies wholly above the threshold iff its end offset < m
        uint32_t c = 0;
#pragma unroll
        for (int e = 0; e < PER_T; ++e) c += gc[kCBuckets - 1 - (tid * PER_T + e)];
        uint32_t tot;
        uint32_t acc = block_exclusive_scan<NT, uint32_t>(c, sh.tmp32, tot);
        uint32_t lm = 0;
#pragma unroll
        for (int e = 0; e < PER_T; ++e) {
            const int d = kCBuckets - 1 - (tid * PER_T + e);
            const uint32_t h = gc[d];
            if (acc < (uint32_t)m && acc + h >= (uint32_t)m) {
                sh.digit = (uint32_t)d;
                sh.above = acc;
            }
            if (acc + h < (uint32_t)m) lm = max(lm, h);
            cur[d] = acc;               // first output slot of bucket d
            acc += h;
        }
        lm = warp_max(lm);
        if ((tid & 31) == 0 && lm) atomicMax(&sh.maxbin, lm);
        __syncthreads();
        if (tid < C) {                  // thread r tells CTA r
            TopkShared *ps = peer<C>(&sh, tid);
            ps->verdict = (sh.maxbin <= (uint32_t)kBinLimit && gc[sh.digit] <= (uint32_t)kCandLimit) ? 1u : 0u;
            ps->bstar = sh.digit;
            ps->above_b = sh.above;
        }
    }
    csync<C>();                         // S3: every CTA knows the verdict
    if (!sh.verdict) {
        if (rank == 0) radix_row();     // a bucket too full for counting
        return;
    }

    // ---- 4. scatter the selected words into CTA 0, grouped by bucket; the
    //         threshold bucket's words into its candidate list
    const int bstar = (int)sh.bstar;
    const uint32_t above = sh.above_b;
    uint64_t *sel0 = peer<C>(sel, 0), *cand0 = peer<C>(cand, 0);
    uint16_t *selb0 = peer<C>(selb, 0);
    uint32_t *slot = cur;               // one CTA: the bucket cursors themselves
    if constexpr (C > 1) {
        // reserve this slice's share of every bucket from the threshold up;
        // its counts become its own cursors
        uint32_t *cur0 = peer<C>(cur, 0);
        for (int j = tid; j < kCBuckets; j += NT) {
            const uint32_t h = hist[j];
            if (j >= bstar && h) hist[j] = atomicAdd(&cur0[j], h);
        }
        __syncthreads();
        slot = hist;
    }
#pragma unroll
    for (int g = 0; g < G; ++g)
        if (tid + g * NT < n4)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int j = (tid + g * NT) * 4 + e;
                if (j < len) {
                    const int b = bucket(v[g][e]);
                    if (b >= bstar) {
                        const uint32_t pos = atomicAdd(&slot[b], 1u);
                        const uint64_t w = ((uint64_t)to_key(v[g][e]) << 32) | (uint32_t)~(uint32_t)(lo + j);
                        if (b > bstar) {
                            sel0[pos] = w;
                            selb0[pos] = (uint16_t)b;
                        } else {
                            cand0[pos - above] = w;
                        }
                    }
                }
            }
    csync<C>();                         // S4: every selected word is in CTA 0
    if (rank != 0) return;

    // ---- 5. CTA 0: rank inside the buckets and write
    auto emit = [&](uint32_t pos, uint64_t w) {
        oidx[pos] = (int32_t)~(uint32_t)w;
        if (oval) oval[pos] = from_key((uint32_t)(w >> 32));
    };
    const uint32_t cstar = gc[bstar];
    const uint32_t need = (uint32_t)m - above;
    for (uint32_t e = tid; e < cstar; e += NT) {
        const uint64_t w = cand[e];
        uint32_t r = 0;
        for (uint32_t q = 0; q < cstar; ++q) r += cand[q] > w;
        if (r < need) emit(above + r, w);
    }
    for (uint32_t p = tid; p < above; p += NT) {
        const uint64_t w = sel[p];
        const int b = selb[p];
        const uint32_t cnt = gc[b], s0 = cur[b] - cnt;   // the cursor ended one bucket past
        uint32_t r = 0;
        for (uint32_t q = s0; q < s0 + cnt; ++q) r += sel[q] > w;
        emit(s0 + r, w);
    }
    pad_row<NT>(oidx, oval, m, k);
}

}  // namespace

size_t topk_smem_bytes(int cap, int kmax)
{
    const size_t cache = (size_t)((cap + 3) & ~3) * 4, pingpong = (size_t)kmax * 8;
    return (size_t)4096 * 4 + (size_t)kmax * 8 + (size_t)kCandLimit * 8 +
           (cache > pingpong ? cache : pingpong);
}

template <int KMAX>
cudaError_t launch_single(const TopkArgs &a, cudaStream_t s)
{
    const size_t smem = topk_smem_bytes(a.cap, a.kmax);
    cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void *>(topk_kernel<KMAX>), (int)smem);
    if (e != cudaSuccess) return e;
    if (a.rows <= 0) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.rows);
    cfg.blockDim = dim3(kTopkThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = a.standalone ? 0 : 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, topk_kernel<KMAX>, a);
}

// Shared memory of one cluster CTA: bucket counts and cursors, the selected
// words and their buckets, and a tail for the candidates and row counts (or
// the radix sort's second buffer).
size_t topk_cluster_smem_bytes(int kmax)
{
    const size_t tail_bucket = (size_t)2 * kCandLimit + kCBuckets, tail_radix = (size_t)2 * kmax;
    return (size_t)2 * kCBuckets * 4 + (size_t)kmax * 10 +
           (tail_bucket > tail_radix ? tail_bucket : tail_radix) * 4;
}

template <int EPT, int KMAX>
cudaError_t launch_cluster(const TopkArgs &a, cudaStream_t s)
{
    auto kern = topk_cluster_kernel<kMaxCluster, kTopkThreads, EPT, KMAX>;
    const size_t smem = topk_cluster_smem_bytes(a.kmax);
    cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void *>(kern), (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)a.rows * kMaxCluster);
    cfg.blockDim = dim3(kTopkThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = a.standalone ? 0 : 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = kMaxCluster;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, a);
}

// Rows that fit one CTA's cache (ld <= a.cap) take one CTA each; longer rows
// a cluster of kMaxCluster CTAs whose threads hold EPT keys each (rows beyond
// kMaxCluster * 512 * 32 keys take the cluster's streamed radix path).
cudaError_t launch_topk(const TopkArgs &a, cudaStream_t s)
{
    if (a.rows <= 0) return cudaSuccess;
    // k up to 2048 (the common case) keeps the radix sort's register rounds
    // small; larger k (up to 8192) takes the wide instances
    const bool big = a.kmax > 2048;
    if (a.ld <= a.cap) return big ? launch_single<8192>(a, s) : launch_single<2048>(a, s);
    const int64_t per_thread = (a.ld + (int64_t)kMaxCluster * kTopkThreads - 1) / ((int64_t)kMaxCluster * kTopkThreads);
    if (per_thread <= 8) return big ? launch_cluster<8, 8192>(a, s) : launch_cluster<8, 2048>(a, s);
    if (per_thread <= 16) return big ? launch_cluster<16, 8192>(a, s) : launch_cluster<16, 2048>(a, s);
    return big ? launch_cluster<32, 8192>(a, s) : launch_cluster<32, 2048>(a, s);
}

}  // namespace li
