// Split-K merge for long contexts (aiknowledge.cn "2.2 PagedAttention 与 KV
// Cache 分页管理" 2.2.4: contexts of 100k tokens assembled from scattered
// blocks).  Each partition p of a sequence's context leaves, per query head,
// its running max m_p (log2 domain, scaled scores), its sum l_p = sum 2^(x-m_p)
// and its unnormalised output o_p = sum 2^(x-m_p) v.  Softmax over the whole
// context is recovered exactly (up to rounding) by
//     M = max_p m_p,  out = sum_p 2^(m_p-M) o_p / sum_p 2^(m_p-M) l_p.
// One warp per (sequence, query head); partitions are merged in index order,
// so the result is deterministic.
#pragma once
#include "attention_common.cuh"

namespace pkv {

struct ReduceParams {
    void* out;                  // [S][Hq][D] of T
    const float* ws_o;          // [S][Hq][maxP][D]
    const float* ws_ml;         // [S][Hq][maxP][2]
    const int32_t* context_lens;
    int S, Hq, D, P, maxP, max_len, bs;
    const int2* member;           // shared-prefix membership, as in AttnParams (nullptr: none)
    const int32_t* query_start;   // chunk mode (non-null): rows are (query row, head), [S + 1]
    int T;
};

// Partials to merge for one output row (0 = the attention kernel wrote it).
// qs: query_start, from global memory or a shared copy.
__device__ __forceinline__ int reduce_count(const ReduceParams& p, int row, const int32_t* qs) {
    const int h_rows = p.Hq;
    if (p.query_start) {  // causal chunk: row = t * Hq + h
        const int t = row / h_rows;
        if (t < qs[0] || t >= qs[p.S]) return 0;
        int lo = 0, hi = p.S;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (qs[mid] <= t) lo = mid;
            else hi = mid;
        }
        int L = p.context_lens[lo];
        L = L < 0 ? 0 : (L > p.max_len ? p.max_len : L);
        const int n = qs[lo + 1] - qs[lo];
        if (n > L) return 0;  // reported by the attention kernel
        if ((L + p.P - 1) / p.P <= 1) return 0;
        const int pos = L - n + (t - qs[lo]);
        return pos / p.P + 1;
    }
    const int s = row / h_rows;
    int L = p.context_lens[s];
    if (L < 0) L = 0;
    if (L > p.max_len) L = p.max_len;
    // A member of a shared-prefix group has ceil(shared/P) prefix partials
    // followed by its own ones (same rule as the attention kernels).
    int shared = 0;
    if (p.member != nullptr) {
        const int2 m = p.member[s];
        if (m.x > 0 && m.y > 0 && m.y <= L) shared = m.y;
    }
    const int nsuf = (L - shared + p.P - 1) / p.P;
    const int nP = (shared + p.P - 1) / p.P + nsuf;
    if (shared == 0 && nP <= 1) return 0;  // written directly by the attention kernel
    return nP;
}

// A CTA handles ROWS (sequence, query head) rows with W warps each.  The
// partitions' maxima are reduced first (M); then warp w of a row sums the
// partitions w, w+W, ... scaled by 2^(m_p - M), each lane owning D/32
// columns, with several partitions' loads in flight; the W partial sums are
// added in warp order through shared memory, so the result does not depend
// on timing.
// Barrier over the W warps of one row (named barrier 1 + row; W > 1 only).
template <int W>
__device__ __forceinline__ void row_sync(int row_in_cta) {
    asm volatile("bar.sync %0, %1;" ::"r"(1 + row_in_cta), "r"(W * 32) : "memory");
}

template <typename T, int D, int W, int ROWS>
__global__ void __launch_bounds__(W * ROWS * 32) splitk_reduce_kernel(const ReduceParams p) {
    constexpr int kPerLane = D / 32;  // 2 or 4 floats
    __shared__ float s_acc_all[ROWS][W][D];
    __shared__ float s_den_all[ROWS][W];
    __shared__ float s_max_all[ROWS][W];
    const int sub = threadIdx.x / (W * 32);  // row of this CTA
    const int row = blockIdx.x * ROWS + sub;  // s * Hq + h
    const int warp = (threadIdx.x >> 5) % W;
    const int lane = threadIdx.x & 31;
    float (&s_acc)[W][D] = s_acc_all[sub];
    float (&s_den)[W] = s_den_all[sub];
    float (&s_max)[W] = s_max_all[sub];
    const int nrows = p.query_start ? p.T * p.Hq : p.S * p.Hq;
    if (row >= nrows) return;  // whole rows return together (W warps of a row)
    const int nP = reduce_count(p, row, p.query_start);
    if (nP == 0) return;
    const int64_t base = (int64_t)row * p.maxP;
    const float* ml = p.ws_ml + base * 2;

    float M = -INFINITY;
    for (int i = warp * 32 + lane; i < nP; i += W * 32) M = fmaxf(M, ml[2 * i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    if (W > 1) {
        if (lane == 0) s_max[warp] = M;
        row_sync<W>(sub);
        M = s_max[0];
#pragma unroll
        for (int w = 1; w < W; ++w) M = fmaxf(M, s_max[w]);
    }

    float acc[kPerLane];
#pragma unroll
    for (int k = 0; k < kPerLane; ++k) acc[k] = 0.f;
    float den = 0.f;
    const float* o = p.ws_o + base * D + lane * kPerLane;
    constexpr int U = 4;  // partitions per batch of loads
    for (int i0 = warp; i0 < nP; i0 += W * U) {
        float wt[U], lp[U], v[U][kPerLane];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = i0 + u * W;
            if (i < nP) {
                const float2 m_l = *reinterpret_cast<const float2*>(ml + 2 * i);
                wt[u] = m_l.x;
                lp[u] = m_l.y;
                if constexpr (kPerLane == 4) {
                    const float4 x = *reinterpret_cast<const float4*>(o + (int64_t)i * D);
                    v[u][0] = x.x; v[u][1] = x.y; v[u][2] = x.z; v[u][3] = x.w;
                } else {
                    const float2 x = *reinterpret_cast<const float2*>(o + (int64_t)i * D);
                    v[u][0] = x.x; v[u][1] = x.y;
                }
            } else {
                wt[u] = -INFINITY;
                lp[u] = 0.f;
#pragma unroll
                for (int k = 0; k < kPerLane; ++k) v[u][k] = 0.f;
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const float w = ex2(wt[u] - M);
            den += w * lp[u];
#pragma unroll
            for (int k = 0; k < kPerLane; ++k) acc[k] += w * v[u][k];
        }
    }
    if (W > 1) {
#pragma unroll
        for (int k = 0; k < kPerLane; ++k) s_acc[warp][lane * kPerLane + k] = acc[k];
        if (lane == 0) s_den[warp] = den;
        row_sync<W>(sub);
        if (warp != 0) return;
    } else {
#pragma unroll
        for (int k = 0; k < kPerLane; ++k) s_acc[0][lane * kPerLane + k] = acc[k];
        if (lane == 0) s_den[0] = den;
        __syncwarp();
    }
    float tot = s_den[0];
#pragma unroll
    for (int w = 1; w < W; ++w) tot += s_den[w];
    const float inv = 1.f / tot;
    T* dst = reinterpret_cast<T*>(p.out) + (int64_t)row * D + lane * kPerLane;
#pragma unroll
    for (int k = 0; k < kPerLane; ++k) {
        float a = s_acc[0][lane * kPerLane + k];
#pragma unroll
        for (int w = 1; w < W; ++w) a += s_acc[w][lane * kPerLane + k];
        dst[k] = static_cast<T>(a * inv);
    }
}

// Few partitions (maxP <= 32): one warp per row, ROWS rows per CTA.  The
// loads that do not depend on the row's partition count go out first -- the
// (m, l) pair of every slot (lane i holds slot i) and, with SPEC >= maxP, the
// partial outputs of every slot -- together with the context length, so a
// row costs one round trip to memory (two without SPEC).  A chunk call's
// query_start is searched in a shared-memory copy when it fits.  Slots past
// the row's count are never used (selected out, so stale values cannot leak
// in); the outputs are summed in slot order, so the result does not depend
// on timing.
constexpr int kReduceIdxMax = 4096;

template <typename T, int D, int ROWS, int SPEC>
__global__ void __launch_bounds__(ROWS * 32) splitk_reduce_warp_kernel(const ReduceParams p) {
    constexpr int KPL = D / 32;  // 2 or 4 floats per lane
    __shared__ int32_t s_idx[kReduceIdxMax];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = blockIdx.x * ROWS + warp;
    const int32_t* qs = p.query_start;
    const int n_idx = p.S + 1;
    if (qs != nullptr && n_idx <= kReduceIdxMax) {  // uniform over the CTA
        for (int i = threadIdx.x; i < n_idx; i += ROWS * 32) s_idx[i] = qs[i];
        __syncthreads();
        qs = s_idx;
    }
    const int nrows = p.query_start ? p.T * p.Hq : p.S * p.Hq;
    if (row >= nrows) return;
    const int64_t base = (int64_t)row * p.maxP;
    const float* o = p.ws_o + base * D + lane * KPL;
    const float2 mlv = lane < p.maxP ? *reinterpret_cast<const float2*>(p.ws_ml + (base + lane) * 2)
                                     : make_float2(-INFINITY, 0.f);
    float v[SPEC > 0 ? SPEC : 1][KPL];
#pragma unroll
    for (int i = 0; i < SPEC; ++i) {
        if (i < p.maxP) {
            if constexpr (KPL == 4) {
                const float4 x = *reinterpret_cast<const float4*>(o + (int64_t)i * D);
                v[i][0] = x.x; v[i][1] = x.y; v[i][2] = x.z; v[i][3] = x.w;
            } else {
                const float2 x = *reinterpret_cast<const float2*>(o + (int64_t)i * D);
                v[i][0] = x.x; v[i][1] = x.y;
            }
        }
    }
    const int nP = reduce_count(p, row, qs);
    if (nP == 0) return;

    float M = lane < nP ? mlv.x : -INFINITY;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    const float w_lane = lane < nP ? ex2(mlv.x - M) : 0.f;
    float den = w_lane * (lane < nP ? mlv.y : 0.f);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);

    float acc[KPL];
#pragma unroll
    for (int k = 0; k < KPL; ++k) acc[k] = 0.f;
    if constexpr (SPEC > 0) {
#pragma unroll
        for (int i = 0; i < SPEC; ++i) {
            const float w = __shfl_sync(0xffffffffu, w_lane, i);
            if (i < nP) {
#pragma unroll
                for (int k = 0; k < KPL; ++k) acc[k] += w * v[i][k];
            }
        }
    } else {
        constexpr int U = 4;  // partitions per batch of loads
        for (int i0 = 0; i0 < nP; i0 += U) {
            float x[U][KPL];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int i = i0 + u < nP ? i0 + u : i0;  // past the count: reload a valid slot, unused
                if constexpr (KPL == 4) {
                    const float4 y = *reinterpret_cast<const float4*>(o + (int64_t)i * D);
                    x[u][0] = y.x; x[u][1] = y.y; x[u][2] = y.z; x[u][3] = y.w;
                } else {
                    const float2 y = *reinterpret_cast<const float2*>(o + (int64_t)i * D);
                    x[u][0] = y.x; x[u][1] = y.y;
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const float w = __shfl_sync(0xffffffffu, w_lane, (i0 + u) & 31);
                if (i0 + u < nP) {
#pragma unroll
                    for (int k = 0; k < KPL; ++k) acc[k] += w * x[u][k];
                }
            }
        }
    }
    const float inv = 1.f / den;
    T* dst = reinterpret_cast<T*>(p.out) + (int64_t)row * D + lane * KPL;
#pragma unroll
    for (int k = 0; k < KPL; ++k) dst[k] = static_cast<T>(acc[k] * inv);
}

}  // namespace pkv
