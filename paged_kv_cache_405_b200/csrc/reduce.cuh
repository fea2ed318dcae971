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
#include "common.cuh"

namespace pkv {

struct ReduceParams {
    void* out;                  // [S][Hq][D] of T
    const float* ws_o;          // [S][Hq][maxP][D]
    const float* ws_ml;         // [S][Hq][maxP][2]
    const int32_t* context_lens;
    int S, Hq, D, P, maxP, max_len, bs;
    const int32_t* group_first;   // shared-prefix groups, as in AttnParams
    const int32_t* group_shared;
    int num_groups;
};

template <typename T, int D>
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const ReduceParams p) {
    constexpr int kPerLane = D / 32;  // 2 or 4 floats
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= p.S * p.Hq) return;
    const int s = warp / p.Hq;
    int L = p.context_lens[s];
    if (L < 0) L = 0;
    if (L > p.max_len) L = p.max_len;
    // Same rule as the attention kernels: a member of a valid shared-prefix
    // group has ceil(shared/P) prefix partials followed by its own ones.
    int shared = 0;
    if (p.num_groups > 0 && s >= p.group_first[0] && s < p.group_first[p.num_groups]) {
        int lo = 0, hi = p.num_groups;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (p.group_first[mid] <= s) lo = mid;
            else hi = mid;
        }
        const int sh = p.group_shared[lo];
        if (sh > 0 && sh % p.bs == 0 && sh <= L) shared = sh;
    }
    const int nsuf = (L - shared + p.P - 1) / p.P;
    const int nP = (shared + p.P - 1) / p.P + nsuf;
    if (shared == 0 && nP <= 1) return;  // written directly by the attention kernel
    const int64_t base = (int64_t)warp * p.maxP;
    const float* ml = p.ws_ml + base * 2;
    float M = -INFINITY;
    for (int i = lane; i < nP; i += 32) M = fmaxf(M, ml[2 * i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float acc[kPerLane];
#pragma unroll
    for (int k = 0; k < kPerLane; ++k) acc[k] = 0.f;
    float den = 0.f;
    const float* o = p.ws_o + base * D + lane * kPerLane;
    for (int i = 0; i < nP; ++i) {
        const float w = ex2(ml[2 * i] - M);
        den += w * ml[2 * i + 1];
        if constexpr (kPerLane == 4) {
            float4 v = *reinterpret_cast<const float4*>(o + (int64_t)i * D);
            acc[0] += w * v.x;
            acc[1] += w * v.y;
            acc[2] += w * v.z;
            acc[3] += w * v.w;
        } else {
            float2 v = *reinterpret_cast<const float2*>(o + (int64_t)i * D);
            acc[0] += w * v.x;
            acc[1] += w * v.y;
        }
    }
    const float inv = 1.f / den;
    T* dst = reinterpret_cast<T*>(p.out) + (int64_t)warp * D + lane * kPerLane;
#pragma unroll
    for (int k = 0; k < kPerLane; ++k) dst[k] = static_cast<T>(acc[k] * inv);
}

}  // namespace pkv
