// Shared-prefix pass on the 5th-generation tensor cores (tcgen05.mma
// kind::f16, accumulators in tensor memory), 16-bit pools, head_dim 128.
//
// Same work and output as prefix_attn_mma_kernel: the queries of a group of
// sequences that share their first tokens in the same physical blocks (a
// system prompt stored once: openeuler.csdn.net PagedAttention explainer 6.1;
// aiknowledge.cn "2.2 PagedAttention 与 KV Cache 分页管理" 2.2.3) attend to
// those shared tokens, one split-K partial (o, m, l) per partition of them,
// merged with each sequence's own partitions by the reduce kernel.  Here a
// CTA of four warps takes 128 query rows of one (group, kv head, partition)
// -- a real dense contraction: every shared K/V tile meets 128 queries.
//
// Per 128-token tile of the shared run (thread t owns query row t = TMEM lane t):
//   S = Q K^T   M = 128 rows, N = 128 tokens, K = 128 head-dim elements (8
//               MMAs of 16).  A = Q (built in shared memory from the rows'
//               query vectors, K-major, 128-byte swizzle, two 64-element
//               column blocks); B = the K tile as loaded by TMA (K-major, the
//               same two blocks).  Two tiles at a time (TMEM columns 0-255).
//   softmax     each thread reads its row of S from TMEM twice: for the
//               maximum over the two tiles, then to write exp2(s - m) as P
//               (the pool's element type) into shared memory (K-major, the
//               A operand of the next product).
//   O += P V    M = 128 rows, N = 128 head-dim elements, K = tokens (16 per
//               MMA).  B = the V tile read MN-major (a token row of 64
//               elements per 128-byte block, the two blocks 16 KB apart).  O
//               stays in TMEM (columns 256-383) across tiles; when a pair
//               of tiles raises a row's maximum, the row is rescaled in TMEM
//               before the pair's products are added.
// Rows are (sequence first + r / G, query head g*G + r % G), as in the mma.sync
// pass; rows whose sequence does not take the group's prefix result (see
// group_members_kernel) get zero queries and no output.
//
// One thread issues the TMA copies and the MMAs; completions arrive on
// mbarriers; every wait is bounded in time, and on a give-up the CTA records
// PKV_DEVERR_TIMEOUT, waits (bounded) for its copies and MMAs in flight,
// frees its tensor memory and returns.  Shared memory (about 225 KB) allows
// one CTA per SM, and a CTA takes 512 TMEM columns, so an allocation never
// waits on another CTA of this kernel.
#pragma once
#include "attention_fp8_tc.cuh"

namespace pkv {

namespace tc {

// Instruction descriptor of kind::f16: T x T -> F32, M = 128, N = 128;
// b_mn: B read MN-major.  T = bf16 (format 1) or f16 (format 0).
template <typename T>
__host__ __device__ constexpr uint32_t idesc_f16_m128_n128(bool b_mn) {
    constexpr uint32_t fmt = std::is_same<T, __half>::value ? 0u : 1u;
    return (1u << 4)                   // D format F32
           | (fmt << 7) | (fmt << 10)  // A, B format
           | (0u << 15)                // A K-major
           | ((b_mn ? 1u : 0u) << 16)  // B major
           | ((128u >> 3) << 17)       // N / 8
           | ((128u >> 4) << 24);      // M / 16
}

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        :
        : "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate ? 1u : 0u)
        : "memory");
}

// 32 consecutive columns of this warp's 32 lanes (thread i: lane base + i).
__device__ __forceinline__ void ld_x32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void st_x32(uint32_t taddr, const float (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
        ::"r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])),
        "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
        "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
        "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])),
        "r"(__float_as_uint(v[17])), "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])),
        "r"(__float_as_uint(v[20])), "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])),
        "r"(__float_as_uint(v[23])), "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])),
        "r"(__float_as_uint(v[26])), "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])),
        "r"(__float_as_uint(v[29])), "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
        : "memory");
}

}  // namespace tc

// Shared memory of the pass (offsets from a 1024-byte aligned base).
struct PrefixTcCfg {
    static constexpr int kBlk = 128 * 128;           // one [128 rows x 128 bytes] swizzled block
    static constexpr int kQOff = 0;                  // Q: 2 blocks (head-dim 0-63, 64-127)
    static constexpr int kKOff = kQOff + 2 * kBlk;   // K ring: 2 tiles x 2 blocks
    static constexpr int kVOff = kKOff + 4 * kBlk;   // V ring: 2 tiles x 2 blocks
    static constexpr int kPOff = kVOff + 4 * kBlk;   // P: 2 tiles x 2 blocks (tokens 0-63, 64-127)
    static constexpr int kBarOff = kPOff + 4 * kBlk; // K full x2, V full x2, S done, O done
    static constexpr int kTmemOff = kBarOff + 8 * 6;
    static constexpr int kSmemBytes = 1024 + kTmemOff + 16;
    static constexpr int kCols = 512;                // S pair: 0-255, O: 256-383
    static constexpr int kColS = 0, kColO = 256;
};

template <typename T>
__global__ void __launch_bounds__(128, 1) prefix_attn_tc_kernel(const AttnParams p,
                                                                const __grid_constant__ CUtensorMap tmK,
                                                                const __grid_constant__ CUtensorMap tmV) {
    using C = PrefixTcCfg;
    constexpr int D = 128, TILE = 128;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tile_r = blockIdx.x;  // 128-row tile of the group
    const int pp = blockIdx.y;      // partition of the shared tokens
    const int gi = blockIdx.z / p.Hkv;
    const int g = blockIdx.z - gi * p.Hkv;
    const int G = p.G;

    int first = p.group_first[gi], last = p.group_first[gi + 1];
    first = max(0, min(first, p.S));
    last = max(first, min(last, p.S));
    if (last - first > p.max_group_size) {
        if (tile_r == 0 && pp == 0 && g == 0 && tid == 0) flag_error(16u /* PKV_DEVERR_GROUP */);
        last = first + p.max_group_size;
    }
    const int rows = (last - first) * G;
    if (tile_r * TILE >= rows) return;  // CTA-uniform
    const int shared = p.group_shared[gi];
    if (shared <= 0 || shared % p.bs != 0 || shared > p.max_len || shared > p.max_shared) return;
    const int t0 = pp * p.P;
    if (t0 >= shared) return;
    const int t1 = min(shared, t0 + p.P);
    const int ntiles = (t1 - t0 + TILE - 1) / TILE;

    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t kfull = sbase + C::kBarOff, vfull = kfull + 16, sbar = kfull + 32, obar = kfull + 40;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kTmemOff);

    // this thread's query row
    const int r = tile_r * TILE + tid;
    const int s_r = first + (r < rows ? r / G : 0);
    const bool live = r < rows && p.member[s_r].x == gi + 1;
    const int h_r = g * G + (r < rows ? r % G : 0);

    // ---- set-up: tensor memory, barriers, Q
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"((uint32_t)C::kCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
    }
    if (tid == 0) {
        prefetch_tensor_map(&tmK);
        prefetch_tensor_map(&tmV);
        for (int i = 0; i < 6; ++i) mbar_init(kfull + 8 * i, 1);
        fence_barrier_init();
    }
    {
        const uint4* qsrc = reinterpret_cast<const uint4*>(reinterpret_cast<const T*>(p.q) +
                                                             ((int64_t)s_r * p.Hq + h_r) * D);
#pragma unroll
        for (int c = 0; c < 16; ++c) {  // 16-byte chunk c: block c / 8, chunk c % 8 of the row
            const uint4 v = live ? qsrc[c] : make_uint4(0u, 0u, 0u, 0u);
            *reinterpret_cast<uint4*>(smem + C::kQOff + (c >> 3) * C::kBlk + tid * 128 + (((c & 7) ^ (tid & 7)) << 4)) = v;
        }
    }
    fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t t_lane = (uint32_t)(warp * 32) << 16;

    // ---- copies: tile i of K (V) into ring slot i % 2 of 2 blocks each; K and
    // V walk the same block-table entries, each with its own window (warp 0)
    const int jb0 = t0 / p.bs;
    BlockWindow kwin, vwin;
    if (warp == 0) {
        kwin.init(p.block_tables + (int64_t)first * p.maxB, jb0, (t1 - 1) / p.bs - jb0 + 1, lane);
        vwin = kwin;
    }
    int kiss = 0, viss = 0;  // tiles whose K / V copies were issued (warp 0), in order
    auto issue = [&](int i, bool is_v, BlockWindow& win) {  // warp 0
        const int tt0 = t0 + i * TILE;
        const int nbox = min(TILE, t1 - tt0) / kTileTok;  // shared runs are whole 16-token boxes
        const uint32_t bar = (is_v ? vfull : kfull) + 8 * (i & 1);
        const uint32_t dst = sbase + (is_v ? C::kVOff : C::kKOff) + (i & 1) * 2 * C::kBlk;
        if (lane == 0) {
            fence_proxy_async();
            mbar_arrive_expect_tx(bar, (uint32_t)(nbox * kTileTok * D * 2));
        }
        for (int j = 0; j < nbox; ++j) {
            const int th = tt0 + j * kTileTok;
            const int blk = win.get(th / p.bs - jb0, lane, p.NB);
            if (lane == 0) {
                const int row = (blk * p.Hkv + g) * p.bs + (th % p.bs);
                const CUtensorMap* map = is_v ? &tmV : &tmK;
                tma_load_2d(dst + j * kTileTok * 128, map, 0, row, bar);
                tma_load_2d(dst + C::kBlk + j * kTileTok * 128, map, 64, row, bar);
            }
        }
        if (is_v) viss = i + 1;
        else kiss = i + 1;
    };
    if (warp == 0) {
        for (int i = 0; i < ntiles && i < 2; ++i) issue(i, false, kwin);
        for (int i = 0; i < ntiles && i < 2; ++i) issue(i, true, vwin);
    }

    constexpr uint32_t kIdS = tc::idesc_f16_m128_n128<T>(false);
    constexpr uint32_t kIdO = tc::idesc_f16_m128_n128<T>(true);
    const float sl2 = p.scale_log2;
    float m = -INFINITY, l = 0.f;
    uint32_t sph = 0, oph = 0;
    bool ok = true, o_started = false;
    int pair = 0;
    for (int a = 0; a < ntiles; a += 2, ++pair) {
        const int nt = min(2, ntiles - a);  // tiles of this pair
        // S = Q K^T for the pair's tiles
        if (tid == 0) {
            for (int u = 0; u < nt && ok; ++u) {
                const int i = a + u;
                ok = mbar_wait(kfull + 8 * (i & 1), (i >> 1) & 1);
                if (!ok) break;
                tc::fence_after_sync();
                const uint32_t kb = sbase + C::kKOff + (i & 1) * 2 * C::kBlk;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    tc::mma_f16(tmem + C::kColS + u * TILE,
                                tc::smem_desc_sw128(sbase + C::kQOff + (kk >> 2) * C::kBlk + (kk & 3) * 32, 16, 1024),
                                tc::smem_desc_sw128(kb + (kk >> 2) * C::kBlk + (kk & 3) * 32, 16, 1024), kIdS, kk > 0);
            }
            if (ok) tc::commit(sbar);
        }
        ok = ok && mbar_wait(sbar, sph);
        sph ^= 1;
        if (!__syncthreads_and(ok ? 1 : 0)) break;
        tc::fence_after_sync();
        // the pair's K slots are free: copy the next pair's K
        if (warp == 0)
            for (int u = 0; u < 2; ++u)
                if (a + 2 + u < ntiles) issue(a + 2 + u, false, kwin);
        // row maximum over the pair's valid tokens
        float pm = -INFINITY;
        for (int u = 0; u < nt; ++u) {
            const int valid = min(TILE, t1 - (t0 + (a + u) * TILE));
            for (int c = 0; c < TILE / 32; ++c) {
                float v[32];
                tc::ld_x32(tmem + t_lane + C::kColS + u * TILE + c * 32, v);
#pragma unroll
                for (int k = 0; k < 32; ++k)
                    if (c * 32 + k < valid) pm = fmaxf(pm, v[k] * sl2);
            }
        }
        const float mn = fmaxf(m, pm);
        const float alpha = ex2(m - mn);  // 0 on the first pair (m = -inf)
        // the previous pair's O products read P and V: wait for them, then
        // rescale the rows whose maximum rose, and refill the V slots
        if (o_started) {
            const bool ook = mbar_wait(obar, oph);
            oph ^= 1;
            if (!__syncthreads_and(ook ? 1 : 0)) { ok = false; break; }
            tc::fence_after_sync();
            if (__any_sync(0xffffffffu, alpha != 1.f)) {
                for (int c = 0; c < D / 32; ++c) {
                    float v[32];
                    tc::ld_x32(tmem + t_lane + C::kColO + c * 32, v);
#pragma unroll
                    for (int k = 0; k < 32; ++k) v[k] *= alpha;
                    tc::st_x32(tmem + t_lane + C::kColO + c * 32, v);
                }
                asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
            }
            if (warp == 0)
                for (int u = 0; u < nt; ++u) issue(a + u, true, vwin);
        }
        l *= alpha;
        m = mn;
        // P = exp2(s - m) in the pool's type, as the A operand of O += P V
        for (int u = 0; u < nt; ++u) {
            const int valid = min(TILE, t1 - (t0 + (a + u) * TILE));
            uint8_t* pb = smem + C::kPOff + u * 2 * C::kBlk;
            for (int c = 0; c < TILE / 32; ++c) {
                float v[32];
                tc::ld_x32(tmem + t_lane + C::kColS + u * TILE + c * 32, v);
                uint32_t w[16];
#pragma unroll
                for (int k = 0; k < 32; k += 2) {
                    const float p0 = c * 32 + k < valid ? ex2(v[k] * sl2 - mn) : 0.f;
                    const float p1 = c * 32 + k + 1 < valid ? ex2(v[k + 1] * sl2 - mn) : 0.f;
                    l += p0 + p1;
                    w[k / 2] = Elt<T>::pack2(p0, p1);
                }
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {  // tokens c*32 + q4*8 .. +7: block, chunk of the row
                    const int tok = c * 32 + q4 * 8;
                    *reinterpret_cast<uint4*>(pb + (tok >> 6) * C::kBlk + tid * 128 + ((((tok & 63) >> 3) ^ (tid & 7)) << 4)) =
                        make_uint4(w[4 * q4], w[4 * q4 + 1], w[4 * q4 + 2], w[4 * q4 + 3]);
                }
            }
        }
        fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        // O += P V over the pair's valid tokens (16 per MMA)
        if (tid == 0) {
            tc::fence_after_sync();
            for (int u = 0; u < nt && ok; ++u) {
                const int i = a + u;
                const int valid = min(TILE, t1 - (t0 + i * TILE));
                ok = mbar_wait(vfull + 8 * (i & 1), (i >> 1) & 1);
                if (!ok) break;
                tc::fence_after_sync();
                const uint32_t vb = sbase + C::kVOff + (i & 1) * 2 * C::kBlk;
                const uint32_t pbase = sbase + C::kPOff + u * 2 * C::kBlk;
                for (int kk = 0; kk < valid / 16; ++kk) {
                    tc::mma_f16(tmem + C::kColO,
                                tc::smem_desc_sw128(pbase + (kk >> 2) * C::kBlk + (kk & 3) * 32, 16, 1024),
                                tc::smem_desc_sw128(vb + kk * 16 * 128, C::kBlk, 1024), kIdO, o_started || kk > 0);
                }
                o_started = true;
            }
            if (ok) tc::commit(obar);
        }
        o_started = true;  // every thread: the pair's products were issued (tid 0) or the CTA gives up below
        ok = __syncthreads_and(ok ? 1 : 0) != 0;
        if (!ok) break;
    }

    bool done = ok;
    if (done) {
        done = mbar_wait(obar, oph);
        done = __syncthreads_and(done ? 1 : 0) != 0;
    }
    if (!done) {  // gave up: let the copies and MMAs in flight finish (bounded), then leave
        if (tid == 0) {
            tc::commit(obar);
            mbar_wait(obar, oph ^ 1);
            mbar_wait(obar, oph);
        }
        if (warp == 0 && lane == 0) {
            for (int i = 0; i < kiss; ++i) mbar_wait(kfull + 8 * (i & 1), (i >> 1) & 1);
            for (int i = 0; i < viss; ++i) mbar_wait(vfull + 8 * (i & 1), (i >> 1) & 1);
        }
        tc::fence_before_sync();
        __syncthreads();
        if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)C::kCols));
        return;
    }
    tc::fence_after_sync();
    // ---- the row's partial: o (unnormalised, at maximum m), m, l
    const int64_t idx = ((int64_t)s_r * p.Hq + h_r) * p.maxP + pp;
    float* dst = p.ws_o + idx * D;
    for (int c = 0; c < D / 32; ++c) {
        float v[32];
        tc::ld_x32(tmem + t_lane + C::kColO + c * 32, v);
        if (live) {
#pragma unroll
            for (int k = 0; k < 32; k += 4)
                *reinterpret_cast<float4*>(dst + c * 32 + k) = make_float4(v[k], v[k + 1], v[k + 2], v[k + 3]);
        }
    }
    if (live) *reinterpret_cast<float2*>(p.ws_ml + idx * 2) = make_float2(m, l);
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)C::kCols));
}

}  // namespace pkv
