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
#include "attention_common.cuh"

namespace pkv {

template <typename T, int D, int WARPS, int STAGES>
struct SimtCfg {
    static constexpr int kRowBytes = D * (int)sizeof(T);
    static constexpr int kTileBytes = kTileTok * kRowBytes;
    static constexpr int kLPT = kRowBytes / 16;       // lanes per token row
    static constexpr int kTPI = 32 / kLPT;            // tokens per pass
    static constexpr int kEPL = 16 / (int)sizeof(T);  // elements per lane
    static constexpr int kPasses = kTileTok / kTPI;
    static constexpr int kStageBytes = 2 * kTileBytes;
    static constexpr int kDataBytes = WARPS * STAGES * kStageBytes;
    static constexpr int kSmemBytes = kDataBytes + WARPS * STAGES * 8;
    static_assert(kLPT >= 1 && kLPT <= 32 && (32 % kLPT) == 0, "row must span 1..32 lanes");
};

template <typename T, int D, int WARPS, int STAGES>
__global__ void __launch_bounds__(WARPS * 32) paged_attn_simt_kernel(const AttnParams p) {
    using C = SimtCfg<T, D, WARPS, STAGES>;
    constexpr int LPT = C::kLPT, TPI = C::kTPI, EPL = C::kEPL;
    extern __shared__ __align__(128) uint8_t smem[];

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int h = blockIdx.x * WARPS + warp;  // query head
    const int part = blockIdx.y;
    const int s = blockIdx.z;
    if (h >= p.Hq) return;

    const Unit u = resolve_unit(p, s, part, part == 0 && h == 0 && lane == 0);
    const int sub = lane / LPT;  // which token of a pass
    const int c = lane % LPT;    // which 16-byte slice of the row
    if (u.t_begin >= u.L) {
        if (part == 0 && u.L == 0 && sub == 0) {  // empty context: zeros
            float z[EPL > 4 ? EPL : 4] = {};
            uint4* o = reinterpret_cast<uint4*>(reinterpret_cast<T*>(p.out) + ((int64_t)s * p.Hq + h) * D) + c;
            *o = Elt<T>::narrow(z);
        }
        return;
    }
    const int t_begin = u.t_begin, t_end = u.t_end;
    const int g = h / p.G;
    const int ntiles = (t_end - t_begin + kTileTok - 1) / kTileTok;

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
        const uint4 qv = reinterpret_cast<const uint4*>(reinterpret_cast<const T*>(p.q) +
                                                        ((int64_t)s * p.Hq + h) * D)[c];
        Elt<T>::widen(qv, qf);
#pragma unroll
        for (int e = 0; e < EPL; ++e) qf[e] *= p.scale_log2;
    }

    const int jb0 = t_begin / p.bs;
    BlockWindow win;
    win.init(p.block_tables + (int64_t)s * p.maxB, jb0, (t_end - 1) / p.bs - jb0 + 1, lane);

    const uint8_t* kp = reinterpret_cast<const uint8_t*>(p.k_pool);
    const uint8_t* vp = reinterpret_cast<const uint8_t*>(p.v_pool);
    auto issue = [&](int i) {
        const int t0 = t_begin + i * kTileTok;
        const int blk = win.get(t0 / p.bs - jb0, lane, p.NB);
        if (lane == 0) {
            const int64_t row = ((int64_t)blk * p.Hkv + g) * p.bs + (t0 % p.bs);
            const int st = i % STAGES;
            const uint32_t bar = bar0 + 8 * st;
            const uint32_t dst = ring_s + st * C::kStageBytes;
            fence_proxy_async();
            mbar_arrive_expect_tx(bar, C::kStageBytes);
            bulk_g2s(dst, kp + row * C::kRowBytes, C::kTileBytes, bar);
            bulk_g2s(dst + C::kTileBytes, vp + row * C::kRowBytes, C::kTileBytes, bar);
        }
    };

    const int npre = ntiles < STAGES ? ntiles : STAGES;
    for (int i = 0; i < npre; ++i) issue(i);

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
        const int valid = min(kTileTok, t_end - (t_begin + i * kTileTok));
        const uint8_t* Ks = ring + st * C::kStageBytes;
        const uint8_t* Vs = Ks + C::kTileBytes;

        float sc[C::kPasses];
#pragma unroll
        for (int ps = 0; ps < C::kPasses; ++ps) {
            const int r = ps * TPI + sub;
            const uint4 kv = *reinterpret_cast<const uint4*>(Ks + r * C::kRowBytes + c * 16);
            float kf[EPL];
            Elt<T>::widen(kv, kf);
            float acc = 0.f;
#pragma unroll
            for (int e = 0; e < EPL; ++e) acc = fmaf(qf[e], kf[e], acc);
#pragma unroll
            for (int off = LPT / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            sc[ps] = r < valid ? acc : -INFINITY;
        }
        float mt = sc[0];
#pragma unroll
        for (int ps = 1; ps < C::kPasses; ++ps) mt = fmaxf(mt, sc[ps]);
#pragma unroll
        for (int off = LPT; off < 32; off <<= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
        const float m_new = fmaxf(m, mt);
        const float alpha = ex2(m - m_new);
        float psum = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) o[e] *= alpha;
#pragma unroll
        for (int ps = 0; ps < C::kPasses; ++ps) {
            const int r = ps * TPI + sub;
            const float pr = ex2(sc[ps] - m_new);
            psum += pr;
            if (r < valid) {
                const uint4 vv = *reinterpret_cast<const uint4*>(Vs + r * C::kRowBytes + c * 16);
                float vf[EPL];
                Elt<T>::widen(vv, vf);
#pragma unroll
                for (int e = 0; e < EPL; ++e) o[e] = fmaf(pr, vf[e], o[e]);
            }
        }
        l = l * alpha + psum;
        m = m_new;
        __syncwarp();
        if (i + STAGES < ntiles) issue(i + STAGES);
    }

    // Combine the token groups of the warp.
#pragma unroll
    for (int off = LPT; off < 32; off <<= 1) {
        l += __shfl_xor_sync(0xffffffffu, l, off);
#pragma unroll
        for (int e = 0; e < EPL; ++e) o[e] += __shfl_xor_sync(0xffffffffu, o[e], off);
    }
    if (sub != 0) return;
    if (u.direct) {
        const float inv = 1.f / l;
        float r[EPL];
#pragma unroll
        for (int e = 0; e < EPL; ++e) r[e] = o[e] * inv;
        uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<T*>(p.out) + ((int64_t)s * p.Hq + h) * D) + c;
        *dst = Elt<T>::narrow(r);
    } else {
        const int64_t idx = ((int64_t)s * p.Hq + h) * p.maxP + u.slot;
        float4* dst = reinterpret_cast<float4*>(p.ws_o + idx * D + c * EPL);
#pragma unroll
        for (int e = 0; e < EPL; e += 4) dst[e / 4] = make_float4(o[e], o[e + 1], o[e + 2], o[e + 3]);
        if (c == 0) *reinterpret_cast<float2*>(p.ws_ml + idx * 2) = make_float2(m, l);
    }
}

}  // namespace pkv
