// Paged decode over FP8 E4M3 pools on the 5th-generation tensor cores
// (tcgen05.mma kind::f8f6f4, accumulators in tensor memory), head_dim 128.
//
// Same work unit as paged_attn_fp8_head_kernel -- one (sequence, query head,
// partition), tokens found block by block through the block table
// (openeuler.csdn.net PagedAttention explainer 4.2; aiknowledge.cn "2.2
// PagedAttention 与 KV Cache 分页管理" 2.2.3-2.2.4) -- but one CTA of four warps
// per unit and 128 tokens per step, and no code is ever widened on the CUDA
// cores: the tensor cores read the E4M3 K and V tiles straight from the
// shared-memory stages TMA filled.
//
// Per 128-token tile (TMEM lane i = MMA row i; thread t of the CTA owns lane t):
//   S^T = K Q^T    M = 128 tokens, N = 16, K = 128 head-dim codes (4 MMAs of
//                  32).  A = the K tile as loaded (K-major, 128-byte swizzle);
//                  B = Q: row 0 = q_hi, row 1 = q_lo, the query scaled by
//                  s_q = 448 / max|q| and split into two E4M3 terms (q s_q =
//                  q_hi + q_lo up to 2^-8 relative), other rows zero.  Thread t
//                  reads columns 0, 1 of lane t: token t's score is
//                  (c0 + c1) / s_q (times the softmax scale and k_scale).
//   softmax        per warp: warp w owns tokens 32w .. 32w+31 of every tile
//                  and keeps its own running maximum m_w and sum l_w (a
//                  split of the context into four interleaved parts, merged
//                  at the end as split-K partials are), so a tile needs no
//                  exchange between warps.
//   O^T = V^T P^T  M = 128 head-dim elements, N = 16, K = tokens (32 per MMA,
//                  one warp's tokens).  A = the V tile read MN-major (a token
//                  row of 128 codes is 128 consecutive M elements); B = P:
//                  rows 2w, 2w+1 = p_hi, p_lo of warp w's tokens (448 p split
//                  into two E4M3 terms like q) and zero elsewhere, so output
//                  columns 2w, 2w+1 collect warp w's tokens only.  Thread t
//                  reads columns 0-7 of lane t and keeps, per warp w,
//                  o_w[t] = o_w[t] * alpha_w + c_2w + c_2w+1 (head-dim element t).
// The splits keep ~8 significant bits of q and of every softmax weight, as
// much as a bf16 operand; K and V codes are used exactly.
//
// Pipeline: one thread issues the TMA copies and the MMAs, and issues the
// next tile's S^T right behind this tile's O^T, so that the two overlap; MMA
// completion arrives on mbarriers (tcgen05.commit); one CTA barrier per tile
// (P written -> O^T issued).  Every wait is bounded in time, and on a give-up
// the CTA records PKV_DEVERR_TIMEOUT, waits (bounded) for its copies and
// MMAs in flight, frees its tensor memory and returns.  Tensor memory: 32
// columns per CTA (S^T in columns 0-15, O^T in 16-31), few enough CTAs per SM
// (shared memory bounds them) that an allocation never waits.
#pragma once
#include "attention_common.cuh"

namespace pkv {

namespace tc {

__device__ __forceinline__ void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor: 128-byte swizzle, the canonical layouts
// of the tcgen05 matrix descriptor (start address, leading / stride byte
// offsets in 16-byte units, descriptor version 1, swizzle mode 2 in bits
// 61-63).  K-major: rows of 128 bytes, 8-row groups SBO apart.  MN-major:
// 128 bytes along M per row, rows of consecutive K, 8-row groups SBO apart.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;  // version
    d |= (uint64_t)2 << 61;  // 128-byte swizzle
    return d;
}

// Instruction descriptor of kind::f8f6f4: E4M3 x E4M3 -> F32, M = 128,
// N = 16; a_mn: A read MN-major.
__host__ __device__ constexpr uint32_t idesc_e4m3_m128_n16(bool a_mn) {
    return (1u << 4)                  // D format F32
           | (0u << 7) | (0u << 10)   // A, B format E4M3
           | ((a_mn ? 1u : 0u) << 15) // A major
           | (0u << 16)               // B K-major
           | ((16u >> 3) << 17)       // N / 8
           | ((128u >> 4) << 24);     // M / 16
}

__device__ __forceinline__ void mma_f8f6f4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                           bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
        :
        : "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate ? 1u : 0u)
        : "memory");
}

// Arrive once on `bar` when every MMA this thread issued so far has completed.
__device__ __forceinline__ void commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// Columns c, c+1 of this warp's 32 lanes (thread i of the warp: lane base + i).
__device__ __forceinline__ void ld_x2(uint32_t taddr, float& a, float& b) {
    uint32_t x, y;
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0, %1}, [%2];" : "=r"(x), "=r"(y) : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
    a = __uint_as_float(x);
    b = __uint_as_float(y);
}

// One E4M3 code of x (round to nearest even, saturating) and its value.
__device__ __forceinline__ uint32_t e4m3_code(float x) { return f32x2_to_e4m3x2(x, 0.f) & 0xffu; }
__device__ __forceinline__ float e4m3_value(uint32_t code) {
    const uint32_t h = e4m3x2_to_f16x2((uint16_t)code);
    return __half2float(__ushort_as_half((unsigned short)(h & 0xffffu)));
}

// Byte offset of element (row r, column c) of a 128-byte-row tile under the
// 128-byte swizzle (16-byte chunk c/16 of row r lands at chunk (c/16) ^ (r & 7)).
__device__ __forceinline__ uint32_t sw128(int r, int c) {
    return (uint32_t)(r * 128 + ((((c >> 4) ^ (r & 7)) << 4) | (c & 15)));
}

}  // namespace tc

constexpr int kTcTile = 128;                   // tokens per step
constexpr int kTcTileBytes = kTcTile * 128;    // one K (or V) tile of codes at head_dim 128
constexpr int kTcColsS = 0, kTcColsO = 16, kTcCols = 32;

template <int STAGES>
struct Fp8TcCfg {
    static constexpr int kStageBytes = 2 * kTcTileBytes;  // K tile, then V tile
    static constexpr int kQOff = STAGES * kStageBytes;    // Q operand: 16 rows x 128 codes
    static constexpr int kPOff = kQOff + 2048;            // P operand: 16 rows x 128 codes
    static constexpr int kBarOff = kPOff + 2048;          // STAGES TMA barriers, S^T and O^T barriers
    static constexpr int kRedOff = kBarOff + 8 * (STAGES + 2);  // 16 floats: alphas (2 x 4), m (4), l (4)
    static constexpr int kTmemOff = kRedOff + 64;         // tensor-memory address
    static constexpr int kSmemBytes = 1024 + kTmemOff + 16;  // + alignment slack
};

#ifndef PKV_FP8_TC_MINB
#define PKV_FP8_TC_MINB 3
#endif

template <int STAGES, typename To>
__global__ void __launch_bounds__(128, PKV_FP8_TC_MINB) paged_attn_fp8_tc_kernel(const AttnParams p,
                                                                                 const __grid_constant__ CUtensorMap tmK,
                                                                                 const __grid_constant__ CUtensorMap tmV) {
    using C = Fp8TcCfg<STAGES>;
    constexpr int D = 128;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.x, part = blockIdx.y, s = blockIdx.z;
    if (h >= p.Hq) return;
    const int g = h / p.G;

    const Unit u = resolve_unit(p, s, part, part == 0 && h == 0 && tid == 0);
    if (u.t_begin >= u.L) {  // CTA-uniform
        if (part == 0 && u.L == 0) reinterpret_cast<To*>(p.out)[((int64_t)s * p.Hq + h) * D + tid] = To(0.f);
        return;
    }
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    uint8_t* qmat = smem + C::kQOff;
    uint8_t* pmat = smem + C::kPOff;
    const uint32_t bar0 = sbase + C::kBarOff;          // TMA stage barriers
    const uint32_t sbar = bar0 + 8 * STAGES;           // S^T completion
    const uint32_t obar = sbar + 8;                    // O^T completion
    float* red = reinterpret_cast<float*>(smem + C::kRedOff);  // [0, 8): alphas by tile parity; [8, 12): m; [12, 16): l
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kTmemOff);

    // ---- set-up: tensor memory, barriers, the Q and P operands
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"((uint32_t)kTcCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
    }
    if (tid == 0) {
        prefetch_tensor_map(&tmK);
        prefetch_tensor_map(&tmV);
        for (int i = 0; i < STAGES + 2; ++i) mbar_init(bar0 + 8 * i, 1);
        fence_barrier_init();
    }
    // every row of Q and P starts at zero; Q rows 0, 1 are written below,
    // P rows 2w, 2w+1 by warp w in its own 32 columns each tile
    for (int i = tid; i < 2 * 2048 / 16; i += 128) *reinterpret_cast<uint4*>(qmat + i * 16) = make_uint4(0u, 0u, 0u, 0u);
    float qv;
    {
        const To* qr = reinterpret_cast<const To*>(p.q) + ((int64_t)s * p.Hq + h) * D;
        qv = static_cast<float>(qr[tid]);
    }
    float amax = fabsf(qv);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if (lane == 0) red[warp] = amax;
    __syncthreads();
    amax = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    const float sq = amax > 0.f ? 448.f / amax : 1.f;
    {
        const float a = qv * sq;
        const uint32_t hi = tc::e4m3_code(a);
        const uint32_t lo = tc::e4m3_code(a - tc::e4m3_value(hi));
        qmat[tc::sw128(0, tid)] = (uint8_t)hi;
        qmat[tc::sw128(1, tid)] = (uint8_t)lo;
    }
    fence_proxy_async();  // generic writes of Q / P before the MMAs read them
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t t_lane = (uint32_t)(warp * 32) << 16;  // this warp's TMEM lanes

    const int t_begin = u.t_begin, t_end = u.t_end;
    const int ntiles = (t_end - t_begin + kTcTile - 1) / kTcTile;
    const int jb0 = t_begin / p.bs;
    BlockWindow win;  // used by warp 0 only
    if (warp == 0) win.init(p.block_tables + (int64_t)s * p.maxB, jb0, (t_end - 1) / p.bs - jb0 + 1, lane);

    int issued = 0;  // tiles whose copies were issued (warp 0)
    auto issue_tma = [&](int i) {  // warp 0
        issued = i + 1;
        const int t0 = t_begin + i * kTcTile;
        const int st = i % STAGES;
        const uint32_t bar = bar0 + 8 * st;
        const uint32_t dst = sbase + st * C::kStageBytes;
        const int nbox = min(kTcTile, t_end - t0 + kTileTok - 1) / kTileTok;  // 16-token boxes of the tile
        if (lane == 0) {
            fence_proxy_async();
            mbar_arrive_expect_tx(bar, (uint32_t)(nbox * 2 * kTileTok * D));
        }
        for (int j = 0; j < nbox; ++j) {
            const int th = t0 + j * kTileTok;
            const int blk = win.get(th / p.bs - jb0, lane, p.NB);
            if (lane == 0) {
                const int row = (blk * p.Hkv + g) * p.bs + (th % p.bs);
                tma_load_2d(dst + j * kTileTok * D, &tmK, 0, row, bar);
                tma_load_2d(dst + kTcTileBytes + j * kTileTok * D, &tmV, 0, row, bar);
            }
        }
    };
    constexpr uint32_t kIdS = tc::idesc_e4m3_m128_n16(false);
    constexpr uint32_t kIdO = tc::idesc_e4m3_m128_n16(true);
    const uint32_t qaddr = sbase + C::kQOff, paddr = sbase + C::kPOff;
    // tid 0: wait for tile i's copies, then S^T(i); false if the wait gave up
    auto issue_s = [&](int i) -> bool {
        const int st = i % STAGES;
        if (!mbar_wait(bar0 + 8 * st, (i / STAGES) & 1)) return false;
        tc::fence_after_sync();
        const uint32_t kaddr = sbase + st * C::kStageBytes;
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk)
            tc::mma_f8f6f4(tmem + kTcColsS, tc::smem_desc_sw128(kaddr + kk * 32, 16, 1024),
                           tc::smem_desc_sw128(qaddr + kk * 32, 16, 1024), kIdS, kk > 0);
        tc::commit(sbar);
        return true;
    };

    if (warp == 0) {
        const int npre = ntiles < STAGES ? ntiles : STAGES;
        for (int i = 0; i < npre; ++i) issue_tma(i);
    }
    bool ok = true;
    if (tid == 0) ok = issue_s(0);

    float m = -INFINITY, lsum = 0.f;        // this warp's running max; this lane's share of its sum
    float o[4] = {0.f, 0.f, 0.f, 0.f};      // head-dim element tid, one partial per warp
    uint32_t sph = 0, oph = 0;
    int i = 0;
    for (; i < ntiles; ++i) {
        const int st = i % STAGES;
        const uint32_t vaddr = sbase + st * C::kStageBytes + kTcTileBytes;
        const int valid = min(kTcTile, t_end - (t_begin + i * kTcTile));
        const int vrows = (valid + 31) & ~31;
        ok = ok && mbar_wait(sbar, sph);  // (tid 0 whose copies gave up does not wait)
        sph ^= 1;
        if (!__syncthreads_and(ok ? 1 : 0)) break;
        tc::fence_after_sync();
        float c0, c1;
        tc::ld_x2(tmem + t_lane + kTcColsS, c0, c1);
        const float x = tid < valid ? (c0 + c1) * (p.scale_log2 / sq) : -INFINITY;
        float wmax = x;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) wmax = fmaxf(wmax, __shfl_xor_sync(0xffffffffu, wmax, off));
        const float mn = fmaxf(m, wmax);
        const float b = mn == -INFINITY ? 0.f : mn;
        const float alpha = ex2(m - b);
        const float pt = ex2(x - b);
        lsum = lsum * alpha + pt;
        m = mn;
        {
            const float a = pt * 448.f;
            const uint32_t hi = tc::e4m3_code(a);
            const uint32_t lo = tc::e4m3_code(a - tc::e4m3_value(hi));
            pmat[tc::sw128(2 * warp, tid)] = (uint8_t)hi;
            pmat[tc::sw128(2 * warp + 1, tid)] = (uint8_t)lo;
        }
        if (lane == 0) red[(i & 1) * 4 + warp] = alpha;
        // V rows past the context inside the last 32-token group may hold any
        // code (NaN included) and would meet a zero weight: the warp owning
        // those tokens clears them (the tile's copies are complete: S^T(i)
        // was issued after them).
        if (valid < vrows && warp == (valid >> 5)) {
            uint8_t* vt = smem + st * C::kStageBytes + kTcTileBytes;
            for (int idx = lane; idx < (vrows - valid) * 8; idx += 32)
                *reinterpret_cast<uint4*>(vt + (valid + idx / 8) * 128 + (idx % 8) * 16) = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        // O^T(i), then S^T(i+1) behind it
        if (tid == 0) {
            tc::fence_after_sync();
            for (int kk = 0; kk < vrows / 32; ++kk)
                tc::mma_f8f6f4(tmem + kTcColsO, tc::smem_desc_sw128(vaddr + kk * 4096, 16, 1024),
                               tc::smem_desc_sw128(paddr + kk * 32, 16, 1024), kIdO, kk > 0);
            tc::commit(obar);
            if (STAGES > 1 && i + 1 < ntiles) ok = issue_s(i + 1);
        }
        const bool ook = mbar_wait(obar, oph);
        oph ^= 1;
        if (!__syncthreads_and(ook ? 1 : 0)) { ok = false; break; }
        tc::fence_after_sync();
        {
            uint32_t c[8];
            asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                         : "=r"(c[0]), "=r"(c[1]), "=r"(c[2]), "=r"(c[3]), "=r"(c[4]), "=r"(c[5]), "=r"(c[6]),
                           "=r"(c[7])
                         : "r"(tmem + t_lane + kTcColsO));
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
            for (int w = 0; w < 4; ++w)
                o[w] = o[w] * red[(i & 1) * 4 + w] + (__uint_as_float(c[2 * w]) + __uint_as_float(c[2 * w + 1]));
        }
        tc::fence_before_sync();
        // the stage of tile i is free (O^T(i) has completed): refill it
        if (warp == 0 && i + STAGES < ntiles) issue_tma(i + STAGES);
        if (STAGES == 1 && tid == 0 && i + 1 < ntiles) ok = issue_s(i + 1);
    }

    if (i < ntiles) {  // gave up: let the copies and MMAs in flight finish (bounded), then leave
        if (tid == 0) {
            tc::commit(obar);
            mbar_wait(obar, oph);
            for (int k = i; k < issued; ++k) mbar_wait(bar0 + 8 * (k % STAGES), (k / STAGES) & 1);
        }
        tc::fence_before_sync();
        __syncthreads();
        if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)kTcCols));
        return;
    }

    // ---- merge the four warps' parts (as split-K partials), output
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, off);
    if (lane == 0) {
        red[8 + warp] = m;
        red[12 + warp] = lsum;
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)kTcCols));
    const float M = fmaxf(fmaxf(red[8], red[9]), fmaxf(red[10], red[11]));
    float ov = 0.f, l = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const float f = ex2(red[8 + w] - M);  // 0 for a warp that saw no token
        ov += f * o[w];
        l += f * red[12 + w];
    }
    ov *= p.v_scale / 448.f;
    const int64_t row = (int64_t)s * p.Hq + h;
    if (u.direct) {
        reinterpret_cast<To*>(p.out)[row * D + tid] = static_cast<To>(ov / l);
    } else {
        const int64_t idx = row * p.maxP + u.slot;
        p.ws_o[idx * D + tid] = ov;
        if (tid == 0) *reinterpret_cast<float2*>(p.ws_ml + idx * 2) = make_float2(M, l);
    }
}

}  // namespace pkv
