// Paged decode attention on CUDA cores: one warp per (sequence, query head,
// partition).  Used for multi-head attention (one query head per kv head),
// where each K/V byte meets one query and the work is a matrix-vector
// product, and as the general fallback (fp32 pools, groups above 16).
//
// What it computes -- softmax(scale q K^T) V over the sequence's cached tokens,
// gathered block by block through the block table (openeuler.csdn.net
// PagedAttention explainer 4.2; aiknowledge.cn "2.2 PagedAttention 与 KV Cache
// 分页管理" 2.2.3-2.2.4) -- with an online softmax in the log2 domain:
//   per 16-token tile:  m' = max(m, max_t x_t);  a = 2^(m - m')
//                       l  = a l + sum_t 2^(x_t - m');  o = a o + sum_t 2^(x_t - m') v_t
//
// Data movement.  The tile of 16 tokens of one (block, kv head) is one
// contiguous run of 16*D elements in the pool, so each stage is two 1-D TMA
// bulk copies (K and V) into this warp's shared-memory ring, completed on an
// mbarrier.  Lane 0 issues; STAGES tiles are in flight per warp and several
// warps per SM keep >50 KB per SM in flight to cover HBM latency.  Block ids
// come from a block-table window the warp loads once per unit (one coalesced
// load of up to 32 entries) and broadcasts with shuffles.
//
// Compute.  LPT = D*sizeof(T)/16 lanes share one token row (16 bytes each);
// the warp handles 32/LPT tokens per pass.  q.k is a 16-byte dot product per
// lane plus a shuffle reduction over the LPT lanes; p.v accumulates per lane
// into its 16-byte slice of the output.  Nothing is written back to shared
// memory, so the ring is read exactly once.
#pragma once
#include <type_traits>

#include "attention_common.cuh"

namespace pkv {

// T: element type of q, out and the pools.
template <typename T, int D, int WARPS, int STAGES, int TILE = kTileTok>
struct SimtCfg {
    static constexpr int kTile = TILE;                 // tokens per pipeline stage
    static constexpr int kRowBytes = D * (int)sizeof(T);
    static constexpr int kTileBytes = TILE * kRowBytes;
    static constexpr int kLPT = kRowBytes / 16;        // lanes per token row
    static constexpr int kTPI = 32 / kLPT;             // tokens per pass
    static constexpr int kEPL = 16 / (int)sizeof(T);  // elements per lane
    static constexpr int kPasses = TILE / kTPI;       // tokens of one lane group per tile
    static_assert(kPasses >= 1 && kPasses * 2 <= kLPT, "tile must give each lane group 1..LPT/2 tokens");
    static constexpr int kStageBytes = 2 * kTileBytes;
    static constexpr int kDataBytes = WARPS * STAGES * kStageBytes;
    static constexpr int kSmemBytes = kDataBytes + WARPS * STAGES * 8;
    static_assert(kLPT >= 1 && kLPT <= 32 && (32 % kLPT) == 0, "row must span 1..32 lanes");
};

// One tile of the CUDA-core kernel (see the kernel below).  FULL = every
// token of the tile is inside the context, so no masking is needed.
template <typename C, typename T, bool FULL>
__device__ __forceinline__ void simt_tile(const uint8_t* Ks, const uint8_t* Vs, int valid, int lane, int sub, int c,
                                          const float (&qf)[C::kEPL], float (&o)[C::kEPL], float& m, float& l) {
    constexpr int LPT = C::kLPT, TPI = C::kTPI, EPL = C::kEPL;
    constexpr int N = C::kPasses;         // tokens of this lane's group in the tile
    constexpr int SPREAD = LPT / N;       // lanes holding each token's score afterwards
    // Partial dot products of this lane's 16-byte slice with each token of its group.
    float v[N];
#pragma unroll
    for (int ps = 0; ps < N; ++ps) {
        const int r = ps * TPI + sub;
        const uint4 kv = *reinterpret_cast<const uint4*>(Ks + r * C::kRowBytes + c * 16);
        float kf[EPL];
        Elt<T>::widen(kv, kf);
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc = fmaf(qf[e], kf[e], acc);
        v[ps] = acc;
    }
    // Butterfly over the LPT lanes of the group: each exchange with a large
    // mask halves the set of tokens a lane keeps (log2 N exchanges), the
    // remaining masks add the halves.  Lane (sub, c) ends with the full score
    // of token j = c / SPREAD of its group.
#pragma unroll
    for (int msk = LPT / 2; msk >= SPREAD; msk >>= 1) {
        const int n = 2 * N * msk / LPT;  // values held before this exchange
        const bool upper = (lane & msk) != 0;
#pragma unroll
        for (int i = 0; i < n / 2; ++i) {
            const float send = upper ? v[i] : v[i + n / 2];
            const float keep = upper ? v[i + n / 2] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, msk);
        }
    }
#pragma unroll
    for (int msk = SPREAD / 2; msk >= 1; msk >>= 1) v[0] += __shfl_xor_sync(0xffffffffu, v[0], msk);
    const int j = c / SPREAD;
    float x = v[0];
    if (!FULL) x = (j * TPI + sub) < valid ? x : -INFINITY;
    float mt = x;
#pragma unroll
    for (int off = SPREAD; off < 32; off <<= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
    const float m_new = fmaxf(m, mt);
    const float alpha = ex2(m - m_new);
    const float pr = ex2(x - m_new);
    l = l * alpha + pr;
    m = m_new;
#pragma unroll
    for (int e = 0; e < EPL; ++e) o[e] *= alpha;
#pragma unroll
    for (int ps = 0; ps < N; ++ps) {
        const int r = ps * TPI + sub;
        const float pw = __shfl_sync(0xffffffffu, pr, sub * LPT + ps * SPREAD);
        uint4 vv = *reinterpret_cast<const uint4*>(Vs + r * C::kRowBytes + c * 16);
        if (!FULL && r >= valid) vv = make_uint4(0u, 0u, 0u, 0u);  // rows past the context may hold NaN
        float vf[EPL];
        Elt<T>::widen(vv, vf);
#pragma unroll
        for (int e = 0; e < EPL; ++e) o[e] = fmaf(pw, vf[e], o[e]);
    }
}

template <typename T, int D, int WARPS, int STAGES, int TILE, bool TENSOR>
__global__ void __launch_bounds__(WARPS * 32, 3) paged_attn_simt_kernel(const AttnParams p,
                                                                       const __grid_constant__ CUtensorMap tmK,
                                                                       const __grid_constant__ CUtensorMap tmV) {
    using C = SimtCfg<T, D, WARPS, STAGES, TILE>;
    constexpr int LPT = C::kLPT, EPL = C::kEPL;
    extern __shared__ __align__(128) uint8_t smem[];

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int h = blockIdx.x * WARPS + warp;  // query head
    int part = blockIdx.y;
    int s = blockIdx.z;
    if (p.lpt) {  // block-collective, before any warp leaves
        const int2 unit = lpt_unit_cta(p, blockIdx.z * gridDim.y + blockIdx.y);
        if (unit.x < 0) return;
        s = unit.x;
        part = unit.y;
    }
    if (h >= p.Hq) return;

    const Unit u = resolve_unit(p, s, part, part == 0 && h == 0 && lane == 0);
    const int sub = lane / LPT;  // which token of a pass
    const int c = lane % LPT;    // which 16-byte slice of the row
    if (u.t_begin >= u.L) {
        if (part == 0 && u.L == 0 && sub == 0) {  // empty context: zeros
            float z[EPL] = {};
            store_slice<T, EPL>(reinterpret_cast<T*>(p.out) + ((int64_t)s * p.Hq + h) * D + c * EPL, z);
        }
        return;
    }
    const int t_begin = u.t_begin, t_end = u.t_end;
    const int g = h / p.G;
    const int ntiles = (t_end - t_begin + TILE - 1) / TILE;

    uint8_t* ring = smem + warp * STAGES * C::kStageBytes;
    const uint32_t ring_s = smem_u32(ring);
    const uint32_t bar0 = smem_u32(smem + C::kDataBytes + warp * STAGES * 8);
    if (lane == 0) {
        for (int i = 0; i < STAGES; ++i) mbar_init(bar0 + 8 * i, 1);
        fence_barrier_init();
    }
    __syncwarp();

    // q slice of this lane, pre-scaled into the log2 domain.
    float qf[EPL];
    {
        load_slice<T, EPL>(reinterpret_cast<const T*>(p.q) + ((int64_t)s * p.Hq + h) * D + c * EPL, qf);
#pragma unroll
        for (int e = 0; e < EPL; ++e) qf[e] *= p.scale_log2;
    }

    const int jb0 = t_begin / p.bs;
    BlockWindow win;
    win.init(p.block_tables + (int64_t)s * p.maxB, jb0, (t_end - 1) / p.bs - jb0 + 1, lane);

    const uint8_t* kp = reinterpret_cast<const uint8_t*>(p.k_pool);
    const uint8_t* vp = reinterpret_cast<const uint8_t*>(p.v_pool);
    auto issue = [&](int i) {
        const int t0 = t_begin + i * TILE;
        const int blk = win.get(t0 / p.bs - jb0, lane, p.NB);
        if (lane == 0) {
            const int64_t row = ((int64_t)blk * p.Hkv + g) * p.bs + (t0 % p.bs);
            const int st = i % STAGES;
            const uint32_t bar = bar0 + 8 * st;
            const uint32_t dst = ring_s + st * C::kStageBytes;
            fence_proxy_async();
            mbar_arrive_expect_tx(bar, C::kStageBytes);
            if constexpr (TENSOR) {  // one (TILE x D) box of the pool viewed as rows of D elements
                tma_load_2d(dst, &tmK, 0, (int)row, bar);
                tma_load_2d(dst + C::kTileBytes, &tmV, 0, (int)row, bar);
            } else {
                bulk_g2s(dst, kp + row * C::kRowBytes, C::kTileBytes, bar);
                bulk_g2s(dst + C::kTileBytes, vp + row * C::kRowBytes, C::kTileBytes, bar);
            }
        }
    };

    const int npre = ntiles < STAGES ? ntiles : STAGES;
    for (int i = 0; i < npre; ++i) issue(i);

    // Running state: m (warp-uniform), a per-lane share of l, and this lane's
    // 16-byte slice of o for the tokens of its group (sub).
    float m = -INFINITY, l = 0.f;
    float o[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) o[e] = 0.f;

    for (int i = 0; i < ntiles; ++i) {
        const int st = i % STAGES;
        const bool ok = mbar_wait(bar0 + 8 * st, (i / STAGES) & 1);
        if (!__all_sync(0xffffffffu, ok)) {
            // Give up on this unit: wait (bounded) for copies still in flight.
            for (int k = i + 1; k < ntiles && k < i + STAGES; ++k) mbar_wait(bar0 + 8 * (k % STAGES), (k / STAGES) & 1);
            return;
        }
        const int valid = min(TILE, t_end - (t_begin + i * TILE));
        const uint8_t* Ks = ring + st * C::kStageBytes;
        const uint8_t* Vs = Ks + C::kTileBytes;
        if (valid == TILE) simt_tile<C, T, true>(Ks, Vs, valid, lane, sub, c, qf, o, m, l);
        else simt_tile<C, T, false>(Ks, Vs, valid, lane, sub, c, qf, o, m, l);
        __syncwarp();
        if (i + STAGES < ntiles) issue(i + STAGES);
    }

    // Combine the token groups of the warp; every token's weight was counted
    // by each of the LPT / kPasses lanes that held its score.
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
    l *= (float)C::kPasses / (float)LPT;
#pragma unroll
    for (int off = LPT; off < 32; off <<= 1) {
#pragma unroll
        for (int e = 0; e < EPL; ++e) o[e] += __shfl_xor_sync(0xffffffffu, o[e], off);
    }
    const int64_t row = (int64_t)s * p.Hq + h;
    if (u.direct) {
        if (sub != 0) return;
        const float inv = 1.f / l;
        float r[EPL];
#pragma unroll
        for (int e = 0; e < EPL; ++e) r[e] = o[e] * inv;
        store_slice<T, EPL>(reinterpret_cast<T*>(p.out) + row * D + c * EPL, r);
        return;
    }
    const unsigned long long seen = p.split_count != nullptr && lane == 0 ? split_peek(p.split_count + row) : 0ull;
    if (sub == 0) {
        const int64_t idx = row * p.maxP + u.slot;
        float4* dst = reinterpret_cast<float4*>(p.ws_o + idx * D + c * EPL);
#pragma unroll
        for (int e = 0; e < EPL; e += 4)
            dst[e / 4] = make_float4(o[e], o[e + 1], o[e + 2], o[e + 3]);
        if (c == 0) *reinterpret_cast<float2*>(p.ws_ml + idx * 2) = make_float2(m, l);
    }
    if (p.split_count != nullptr) merge_if_last<T, D>(p, row, u.nsuf, lane, seen);
}

}  // namespace pkv
