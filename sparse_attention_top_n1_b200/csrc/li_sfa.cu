// li_sfa.cu -- sparse attention over the indexer's selected keys.
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
// row, each taking a share of its keys), one warp per 16 heads.  The row's
// selected keys are taken 64 at a time: their K and V rows are gathered from
// wherever the index points (BSND, TND or a paged pool) into shared memory
// with 16-byte cp.async copies, double-buffered against the math; S = Q K^T
// and O += P V run on the tensor cores (m16n8k16, fp32 accumulation) with the
// softmax kept online in registers (running max and sum per head, the
// FlashAttention recurrence), so the selected keys are read once and nothing
// but the output is written.  The weights enter P V rounded to the input
// type and the normaliser sums the same rounded values.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cooperative_groups.h>

#include <cmath>
#include <cstdio>
#include <cstdint>

#include "li.h"

namespace li {
li_status report_error(li_status s, const char *msg);
void set_launch_count(int32_t n);
cudaError_t set_max_dynamic_smem(const void *kern, int bytes);
}  // namespace li

namespace {

constexpr int kTile = 64;                 // selected keys per tile
constexpr int kHd = 128;                  // D = Dv
constexpr int kRowBytes = kHd * 2;        // one key or value row
constexpr int kChunks = kRowBytes / 16;   // 16-byte chunks per row
constexpr int kTileBytes = kTile * kRowBytes;
constexpr int kRowMapBytes = 2 * kTile * 4;    // [2][kTile] key row of each slot
constexpr int kMergeBytes = 2 * 128 * 4;       // a cluster's per-head (max, sum) partials
constexpr int kMaskBytes = 16;                 // [2][2] slot-validity bits
constexpr int kSmem = 4 * kTileBytes + kRowMapBytes + kMergeBytes + kMaskBytes + 128;
constexpr int kMaxSplit = 8;             // CTAs (one cluster) sharing a row's keys

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
};

__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte global->shared copy; src_bytes = 0 fills the destination with zeros
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

template <bool F16>
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    if constexpr (F16)
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    else
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

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

// Byte offset of 16-byte chunk `ch` of row `r` in a tile: rows of 256 B, the
// low three bits of the chunk index XOR-ed with the row so that the eight
// rows an ldmatrix phase reads sit in eight different bank groups.
__device__ __forceinline__ uint32_t tile_off(int r, int ch)
{
    return (uint32_t)(r * kRowBytes + ((ch ^ (r & 7)) << 4));
}

__device__ __forceinline__ int32_t clampi(int64_t v, int64_t lo, int64_t hi)
{
    return (int32_t)(v < lo ? lo : (v > hi ? hi : v));
}

// C > 1: a cluster of C CTAs shares one row; CTA `part` takes its share of the
// row's key tiles, and the C partial (max, sum, O) triples are merged through
// distributed shared memory, so no global scratch is needed.
template <int NW, bool F16, int C>
__global__ void __launch_bounds__(32 * NW) sfa_kernel(const SfaArgs a)
{
    static_assert(kChunks == 16, "row chunk arithmetic assumes 256-byte rows");
    constexpr int NT = 32 * NW;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    uint8_t *sK = base;                                      // [2] key tiles
    uint8_t *sV = base + 2 * kTileBytes;                     // [2] value tiles
    int32_t *sRow = reinterpret_cast<int32_t *>(base + 4 * kTileBytes);   // [2][kTile] key row, -1 = none
    uint32_t *sMask = reinterpret_cast<uint32_t *>(base + 4 * kTileBytes + kRowMapBytes + kMergeBytes);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, c = lane & 3;
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

    // ---- this warp's 16 heads of the query as m16n8k16 A fragments
    uint32_t qf[8][4];
    {
        const uint16_t *qh = a.q + ((int64_t)row * a.N1 + warp * 16) * kHd;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const int d = kk * 16 + 2 * c;
            qf[kk][0] = *reinterpret_cast<const uint32_t *>(qh + g * kHd + d);
            qf[kk][1] = *reinterpret_cast<const uint32_t *>(qh + (g + 8) * kHd + d);
            qf[kk][2] = *reinterpret_cast<const uint32_t *>(qh + g * kHd + d + 8);
            qf[kk][3] = *reinterpret_cast<const uint32_t *>(qh + (g + 8) * kHd + d + 8);
        }
    }

    const int32_t *irow = a.idx + (int64_t)row * a.K;
    // slot r of tile t: the key/value row its index names, or -1
    auto resolve = [&](int t, int buf) -> int {
        int ok = 0;
        for (int r = tid; r < kTile; r += NT) {    // one CTA may have fewer threads than slots
            const int j = t * kTile + r;
            int kr = -1;
            if (j < a.K) {
                const int e = irow[j];
                if (e >= 0 && e < Sk) {
                    if (a.layout_kv == LI_PA_BSND) {
                        const int id = a.block_table[(int64_t)b * a.max_blocks_per_seq + e / a.block_size];
                        if (id >= 0 && id < a.num_blocks) kr = id * a.block_size + e % a.block_size;
                        else if (a.status) atomicOr(a.status, LI_DEV_BAD_BLOCK);
                    } else {
                        kr = (int)(k_off + e);
                    }
                } else if (e != -1 && a.status) {
                    atomicOr(a.status, LI_DEV_BAD_INDEX);
                }
            }
            sRow[buf * kTile + r] = kr;
            ok |= kr >= 0;
            // whole warps run this loop (kTile is a multiple of 32)
            const unsigned bal = __ballot_sync(0xffffffffu, kr >= 0);
            if ((r & 31) == 0) sMask[buf * 2 + (r >> 5)] = bal;
        }
        return ok;
    };
    // gather the tile's key and value rows (zeros for empty slots)
    auto issue = [&](int buf) {
        const uint32_t kd = smem_addr(sK + buf * kTileBytes), vd = smem_addr(sV + buf * kTileBytes);
        for (int ci = tid; ci < kTile * kChunks; ci += NT) {
            const int r = ci >> 4, ch = ci & 15;
            const int kr = sRow[buf * kTile + r];
            const int64_t off = (int64_t)(kr < 0 ? 0 : kr) * kHd + ch * 8;
            const uint32_t n = kr < 0 ? 0u : 16u;
            cp_async16(kd + tile_off(r, ch), a.k + off, n);
            cp_async16(vd + tile_off(r, ch), a.v + off, n);
        }
        cp_async_commit();
    };

    float o[16][4];
#pragma unroll
    for (int dn = 0; dn < 16; ++dn) o[dn][0] = o[dn][1] = o[dn][2] = o[dn][3] = 0.f;
    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};

    const int nt_all = valid_row ? (a.K + kTile - 1) / kTile : 0;
    const int t_begin = nt_all * part / C, t_end = nt_all * (part + 1) / C;
    int any_cur = 0;
    if (t_begin < t_end) {
        any_cur = __syncthreads_or(resolve(t_begin, 0));
        if (any_cur) issue(0);
        else cp_async_commit();
    }
    for (int t = t_begin; t < t_end; ++t) {
        const int buf = (t - t_begin) & 1;
        int any_next = 0;
        if (t + 1 < t_end) {
            any_next = __syncthreads_or(resolve(t + 1, buf ^ 1));
            if (any_next) issue(buf ^ 1);
            else cp_async_commit();
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        if (any_cur) {
            const uint32_t kb = smem_addr(sK + buf * kTileBytes), vb = smem_addr(sV + buf * kTileBytes);
            const uint64_t valid = (uint64_t)sMask[buf * 2] | ((uint64_t)sMask[buf * 2 + 1] << 32);
            // S = Q K^T for 16 heads x 64 keys
            float s[8][4];
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
                for (int np = 0; np < 4; ++np) {
                    const int key = np * 16 + (lane & 7) + ((lane >> 4) << 3);
                    const int ch = kk * 2 + ((lane >> 3) & 1);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(kb + tile_off(key, ch), b0, b1, b2, b3);
                    mma16816<F16>(s[2 * np], qf[kk], b0, b1);
                    mma16816<F16>(s[2 * np + 1], qf[kk], b2, b3);
                }
            }
            // online softmax in the log2 domain; rows g (e = 0, 1) and g + 8 (e = 2, 3)
            float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const bool ok = (valid >> (nt * 8 + 2 * c + (e & 1))) & 1u;
                    s[nt][e] = ok ? s[nt][e] * a.scale_log2 : -INFINITY;
                    mx[e >> 1] = fmaxf(mx[e >> 1], s[nt][e]);
                }
            float base_[2], alpha[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
                mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
                const float mn = fmaxf(m[h], mx[h]);
                base_[h] = mn == -INFINITY ? 0.f : mn;
                alpha[h] = exp2f(m[h] - base_[h]);
                m[h] = mn;
            }
            // the weights, rounded to dtype as the P.V product sees them, packed
            // straight into A fragments; the normaliser sums the same values
            float rs[2] = {0.f, 0.f};
            uint32_t pk[8][2];
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    pk[nt][h] = pack2<F16>(exp2f(s[nt][2 * h] - base_[h]), exp2f(s[nt][2 * h + 1] - base_[h]));
                    rs[h] += unpack_lo<F16>(pk[nt][h]) + unpack_hi<F16>(pk[nt][h]);
                }
#pragma unroll
            for (int h = 0; h < 2; ++h) l[h] = l[h] * alpha[h] + rs[h];
            // the running max moved for some head of this warp: rescale O
            if (__any_sync(0xffffffffu, alpha[0] != 1.f || alpha[1] != 1.f)) {
#pragma unroll
                for (int dn = 0; dn < 16; ++dn) {
                    o[dn][0] *= alpha[0];
                    o[dn][1] *= alpha[0];
                    o[dn][2] *= alpha[1];
                    o[dn][3] *= alpha[1];
                }
            }
            // O += P V
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t pa[4] = {pk[2 * j][0], pk[2 * j][1], pk[2 * j + 1][0], pk[2 * j + 1][1]};
#pragma unroll
                for (int dp = 0; dp < 8; ++dp) {
                    const int key = j * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
                    const int ch = dp * 2 + (lane >> 4);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(vb + tile_off(key, ch), b0, b1, b2, b3);
                    mma16816<F16>(o[2 * dp], pa, b0, b1);
                    mma16816<F16>(o[2 * dp + 1], pa, b2, b3);
                }
            }
        }
        __syncthreads();                       // the buffers of tile t are refilled next
        any_cur = any_next;
    }

    // ---- normalise and store (zeros and -inf when nothing was selected)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        l[h] += __shfl_xor_sync(0xffffffffu, l[h], 1);
        l[h] += __shfl_xor_sync(0xffffffffu, l[h], 2);
    }
    if constexpr (C > 1) {
        // partials into this CTA's shared memory (the tile buffers are free)
        float *sO = reinterpret_cast<float *>(base);                 // [N1][128], unnormalised
        float *sM = reinterpret_cast<float *>(base + 4 * kTileBytes + kRowMapBytes);    // [N1]
        float *sL = sM + 128;                                        // [N1]
        const int h0 = warp * 16 + g, h1 = h0 + 8;
#pragma unroll
        for (int dn = 0; dn < 16; ++dn) {
            const int d = dn * 8 + 2 * c;
            sO[h0 * kHd + d] = o[dn][0];
            sO[h0 * kHd + d + 1] = o[dn][1];
            sO[h1 * kHd + d] = o[dn][2];
            sO[h1 * kHd + d + 1] = o[dn][3];
        }
        if (c == 0) {
            sM[h0] = m[0];
            sL[h0] = l[0];
            sM[h1] = m[1];
            sL[h1] = l[1];
        }
        cooperative_groups::cluster_group cl = cooperative_groups::this_cluster();
        cl.sync();
        // CTA `part` merges heads [part*N1/C, (part+1)*N1/C) over the C partials
        const int hpc = a.N1 / C;
        const float ln2 = 0.69314718055994531f;
        for (int e = tid; e < hpc * kHd; e += NT) {
            const int h = part * hpc + e / kHd, d = e % kHd;
            float M = -INFINITY;
#pragma unroll
            for (int r = 0; r < C; ++r) M = fmaxf(M, cl.map_shared_rank(sM, r)[h]);
            float L = 0.f, O = 0.f;
            if (M != -INFINITY) {
#pragma unroll
                for (int r = 0; r < C; ++r) {
                    const float mr = cl.map_shared_rank(sM, r)[h];
                    if (mr == -INFINITY) continue;
                    const float w = exp2f(mr - M);
                    L += cl.map_shared_rank(sL, r)[h] * w;
                    O += cl.map_shared_rank(sO, r)[h * kHd + d] * w;
                }
            }
            const float v = L > 0.f ? O / L : 0.f;
            a.out[((int64_t)row * a.N1 + h) * kHd + d] =
                F16 ? __half_as_ushort(__float2half_rn(v)) : __bfloat16_as_ushort(__float2bfloat16_rn(v));
            if (d == 0 && a.lse) a.lse[(int64_t)row * a.N1 + h] = L > 0.f ? (M + log2f(L)) * ln2 : -INFINITY;
        }
        cl.sync();                             // every peer has read this CTA's partials
        return;
    }
    const float inv0 = l[0] > 0.f ? 1.f / l[0] : 0.f, inv1 = l[1] > 0.f ? 1.f / l[1] : 0.f;
    uint16_t *orow = a.out + ((int64_t)row * a.N1 + warp * 16) * kHd;
#pragma unroll
    for (int dn = 0; dn < 16; ++dn) {
        const int d = dn * 8 + 2 * c;
        *reinterpret_cast<uint32_t *>(orow + g * kHd + d) = pack2<F16>(o[dn][0] * inv0, o[dn][1] * inv0);
        *reinterpret_cast<uint32_t *>(orow + (g + 8) * kHd + d) = pack2<F16>(o[dn][2] * inv1, o[dn][3] * inv1);
    }
    if (a.lse && c == 0) {
        const float ln2 = 0.69314718055994531f;
        float *lr = a.lse + (int64_t)row * a.N1 + warp * 16;
        lr[g] = l[0] > 0.f ? (m[0] + log2f(l[0])) * ln2 : -INFINITY;
        lr[g + 8] = l[1] > 0.f ? (m[1] + log2f(l[1])) * ln2 : -INFINITY;
    }
}

template <int NW, bool F16, int C>
cudaError_t launch(const SfaArgs &a, int rows, cudaStream_t s)
{
    auto kern = sfa_kernel<NW, F16, C>;
    cudaError_t e = li::set_max_dynamic_smem(reinterpret_cast<const void *>(kern), kSmem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)rows * C);
    cfg.blockDim = dim3(32 * NW);
    cfg.dynamicSmemBytes = kSmem;
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

template <int NW, bool F16>
cudaError_t launch_split(const SfaArgs &a, int rows, int split, cudaStream_t s)
{
    switch (split) {
    case 1: return launch<NW, F16, 1>(a, rows, s);
    case 2: return launch<NW, F16, 2>(a, rows, s);
    case 4: return launch<NW, F16, 4>(a, rows, s);
    case 8: return launch<NW, F16, 8>(a, rows, s);
    }
    return cudaErrorInvalidValue;
}

template <bool F16>
cudaError_t launch_nw(const SfaArgs &a, int rows, int split, cudaStream_t s)
{
    switch (a.N1) {
    case 16: return launch_split<1, F16>(a, rows, split, s);
    case 32: return launch_split<2, F16>(a, rows, split, s);
    case 64: return launch_split<4, F16>(a, rows, split, s);
    case 128: return launch_split<8, F16>(a, rows, split, s);
    }
    return cudaErrorInvalidValue;
}

// CTAs per row: enough to give every SM two rows' worth of work when rows are
// few (decode), at least one 64-key tile per CTA, a power of two up to 8.
int choose_split(int64_t rows, int K, int sms)
{
    const int ntiles = (K + kTile - 1) / kTile;
    int c = 1;
    while (c < kMaxSplit && rows * c < 2LL * sms && 2 * c <= ntiles) c *= 2;
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
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int split = choose_split(rows, a.K, sms);
    const cudaError_t e = p->dtype == LI_FP16 ? launch_nw<true>(a, (int)rows, split, s)
                                              : launch_nw<false>(a, (int)rows, split, s);
    if (e != cudaSuccess) {
        char msg[200];
        snprintf(msg, sizeof msg, "li_sparse_attention: launch failed (%s)", cudaGetErrorString(e));
        return report_error(LI_ERR_CUDA, msg);
    }
    li::set_launch_count(1);
    return LI_OK;
}
