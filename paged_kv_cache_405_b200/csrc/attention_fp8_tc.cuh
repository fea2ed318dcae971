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
//   softmax        each thread owns one token; the tile maximum and, at the
//                  end, the sum go through shared memory across the 4 warps.
//   O^T = V^T P^T  M = 128 head-dim elements, N = 16, K = tokens (32 per MMA).
//                  A = the V tile read MN-major (a token row of 128 codes is
//                  128 consecutive M elements); B = P: row 0 = p_hi, row 1 =
//                  p_lo, 448 p split into two E4M3 terms like q.  The tile's
//                  O^T is written fresh into TMEM; thread t reads columns 0,
//                  1 of lane t and accumulates o[t] = o[t] * alpha + c0 + c1
//                  in a register (head-dim element t).
// The splits keep ~8 significant bits of q and of every softmax weight, as
// much as a bf16 operand; K and V codes are used exactly.
//
// Synchronisation: one thread issues the TMA copies and the MMAs; MMA
// completion arrives on an mbarrier (tcgen05.commit); every wait is bounded
// in time, and on a give-up the CTA records PKV_DEVERR_TIMEOUT, waits
// (bounded) for its copies and MMAs in flight, frees its tensor memory and
// returns.  Tensor memory: 32 columns per CTA (S^T in columns 0-15, O^T in
// 16-31), at most 3 CTAs per SM (shared memory), so an allocation never waits.
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
    static constexpr int kBarOff = kPOff + 2048;          // STAGES TMA barriers, then the MMA barrier
    static constexpr int kRedOff = kBarOff + 8 * (STAGES + 1);  // 4 floats of block reductions
    static constexpr int kTmemOff = kRedOff + 16;         // tensor-memory address
    static constexpr int kSmemBytes = 1024 + kTmemOff + 16;  // + alignment slack
};

template <int STAGES, typename To>
__global__ void __launch_bounds__(128, 3) paged_attn_fp8_tc_kernel(const AttnParams p,
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
    const uint32_t mbar = bar0 + 8 * STAGES;           // MMA completion barrier
    float* red = reinterpret_cast<float*>(smem + C::kRedOff);
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
        for (int i = 0; i <= STAGES; ++i) mbar_init(bar0 + 8 * i, 1);
        fence_barrier_init();
    }
    // rows 2..15 of Q and P stay zero; rows 0, 1 are written below / per tile
    for (int i = tid; i < 2 * 2048 / 16; i += 128) {
        const int off = i < 128 ? i * 16 : 2048 + (i - 128) * 16;
        *reinterpret_cast<uint4*>(qmat + off) = make_uint4(0u, 0u, 0u, 0u);
    }
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
    fence_proxy_async();  // generic writes of Q / P zeros before the MMAs read them
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

    auto issue = [&](int i) {  // warp 0
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
    if (warp == 0) {
        const int npre = ntiles < STAGES ? ntiles : STAGES;
        for (int i = 0; i < npre; ++i) issue(i);
    }

    constexpr uint32_t kIdS = tc::idesc_e4m3_m128_n16(false);
    constexpr uint32_t kIdO = tc::idesc_e4m3_m128_n16(true);
    const uint32_t qaddr = sbase + C::kQOff, paddr = sbase + C::kPOff;
    float m = -INFINITY, lpart = 0.f, o = 0.f;
    uint32_t mphase = 0;
    bool ok = true;
    int i = 0;
    for (; i < ntiles; ++i) {
        const int st = i % STAGES;
        const uint32_t kaddr = sbase + st * C::kStageBytes, vaddr = kaddr + kTcTileBytes;
        const int valid = min(kTcTile, t_end - (t_begin + i * kTcTile));
        ok = mbar_wait(bar0 + 8 * st, (i / STAGES) & 1);
        if (!__syncthreads_and(ok ? 1 : 0)) break;
        // V rows past the context inside the last 32-token group may hold any
        // code (NaN included) and would meet a zero weight: clear them.
        const int vrows = (valid + 31) & ~31;
        if (valid < vrows) {
            uint8_t* vt = smem + st * C::kStageBytes + kTcTileBytes;
            for (int idx = tid; idx < (vrows - valid) * 8; idx += 128)
                *reinterpret_cast<uint4*>(vt + (valid + idx / 8) * 128 + (idx % 8) * 16) = make_uint4(0u, 0u, 0u, 0u);
            fence_proxy_async();
        }
        __syncthreads();
        // S^T = K Q^T
        if (tid == 0) {
            tc::fence_after_sync();
#pragma unroll
            for (int kk = 0; kk < D / 32; ++kk)
                tc::mma_f8f6f4(tmem + kTcColsS, tc::smem_desc_sw128(kaddr + kk * 32, 16, 1024),
                               tc::smem_desc_sw128(qaddr + kk * 32, 16, 1024), kIdS, kk > 0);
            tc::commit(mbar);
        }
        ok = mbar_wait(mbar, mphase);
        mphase ^= 1;
        if (!__syncthreads_and(ok ? 1 : 0)) break;
        tc::fence_after_sync();
        float c0, c1;
        tc::ld_x2(tmem + t_lane + kTcColsS, c0, c1);
        const float x = tid < valid ? (c0 + c1) * (p.scale_log2 / sq) : -INFINITY;
        float tmax = x;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, off));
        if (lane == 0) red[warp] = tmax;
        __syncthreads();
        tmax = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
        const float mn = fmaxf(m, tmax);
        const float b = mn == -INFINITY ? 0.f : mn;
        const float alpha = ex2(m - b);
        const float pt = ex2(x - b);
        lpart = lpart * alpha + pt;
        m = mn;
        {
            const float a = pt * 448.f;
            const uint32_t hi = tc::e4m3_code(a);
            const uint32_t lo = tc::e4m3_code(a - tc::e4m3_value(hi));
            pmat[tc::sw128(0, tid)] = (uint8_t)hi;
            pmat[tc::sw128(1, tid)] = (uint8_t)lo;
        }
        fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        // O^T = V^T P^T over the tile's 32-token groups that hold tokens
        if (tid == 0) {
            tc::fence_after_sync();
            for (int kk = 0; kk < vrows / 32; ++kk)
                tc::mma_f8f6f4(tmem + kTcColsO, tc::smem_desc_sw128(vaddr + kk * 4096, 16, 1024),
                               tc::smem_desc_sw128(paddr + kk * 32, 16, 1024), kIdO, kk > 0);
            tc::commit(mbar);
        }
        ok = mbar_wait(mbar, mphase);
        mphase ^= 1;
        if (!__syncthreads_and(ok ? 1 : 0)) break;
        tc::fence_after_sync();
        float d0, d1;
        tc::ld_x2(tmem + t_lane + kTcColsO, d0, d1);
        o = o * alpha + (d0 + d1);
        tc::fence_before_sync();
        __syncthreads();  // the stage, S, O and P are free for the next tile
        if (warp == 0 && i + STAGES < ntiles) issue(i + STAGES);
    }

    if (i < ntiles) {  // gave up: let the copies and MMAs in flight finish (bounded), then leave
        if (tid == 0) {
            tc::commit(mbar);
            mbar_wait(mbar, mphase);
            for (int k = i; k < ntiles && k < i + STAGES; ++k) mbar_wait(bar0 + 8 * (k % STAGES), (k / STAGES) & 1);
        }
        tc::fence_before_sync();
        __syncthreads();
        if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)kTcCols));
        return;
    }

    // ---- sum of the weights, output
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) lpart += __shfl_xor_sync(0xffffffffu, lpart, off);
    if (lane == 0) red[warp] = lpart;
    tc::fence_before_sync();
    __syncthreads();
    const float l = (red[0] + red[1]) + (red[2] + red[3]);
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)kTcCols));
    const float ov = o * (p.v_scale / 448.f);
    const int64_t row = (int64_t)s * p.Hq + h;
    if (u.direct) {
        reinterpret_cast<To*>(p.out)[row * D + tid] = static_cast<To>(ov / l);
    } else {
        const int64_t idx = row * p.maxP + u.slot;
        p.ws_o[idx * D + tid] = ov;
        if (tid == 0) *reinterpret_cast<float2*>(p.ws_ml + idx * 2) = make_float2(m, l);
    }
}

}  // namespace pkv
