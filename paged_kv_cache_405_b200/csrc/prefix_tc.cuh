// Shared-prefix pass on the 5th-generation tensor cores (tcgen05.mma
// kind::f16, accumulators in tensor memory), 16-bit pools, head_dim 128.
//
// Same work and output as prefix_attn_mma_kernel: the queries of a group of
// sequences that share their first tokens in the same physical blocks (a
// system prompt stored once: openeuler.csdn.net PagedAttention explainer 6.1;
// aiknowledge.cn "2.2 PagedAttention 与 KV Cache 分页管理" 2.2.3) attend to
// those shared tokens, one split-K partial (o, m, l) per partition of them,
// merged with each sequence's own partitions by the reduce kernel.  Here one
// CTA takes QT tiles of 128 query rows of one (group, kv head, partition) --
// a real dense contraction: every shared K/V tile meets 128 * QT queries.
//
// Per 64-token tile j of the partition and Q tile q (thread t of softmax
// warpgroup q owns query row t = TMEM lane t):
//   S = Q K^T   M = 128 rows, N = 64 tokens, K = 128 head-dim elements (8
//               MMAs of 16).  A = Q (built in shared memory from the rows'
//               query vectors, K-major, 128-byte swizzle, two 64-element
//               column blocks); B = the K tile as TMA loads it (K-major, the
//               same two blocks).  S goes to one of two TMEM buffers, so the
//               next tile's S is computed while this one's softmax runs.
//   softmax     the thread reads its 64 scores and writes P = exp2(s - m) in
//               the pool's element type back over them in tensor memory (two
//               values per 32-bit column).  m is a reference maximum: it
//               moves (and O and l are rescaled by exp2(m_old - m_new)) only
//               when a tile's maximum exceeds it by more than 8, so P stays
//               below 2^8 and O is rarely touched; o, l and m stay one
//               consistent partial, whose value is the softmax's exactly.
//   O += P V    M = 128 rows, N = 128 head-dim elements, K = tokens (16 per
//               MMA).  A = P read from tensor memory; B = the V tile read
//               MN-major (a token row of 64 elements per 128-byte row, the
//               two head-dim blocks kHalf bytes apart).  O stays in TMEM.
// Rows are (sequence first + r / G, query head g*G + r % G), as in the mma.sync
// pass; rows whose sequence does not take the group's prefix result (see
// group_members_kernel) get zero queries and no output.
//
// Warp roles: warps 0 .. 4*QT-1 are the softmax warpgroups (warp w reads TMEM
// lanes 32*(w % 4) ..), then one warp issues the K copies, one the V copies
// (each into its own ring of KS / VS tiles, refilled as the MMAs release
// slots), and lane 0 of the last warp issues every MMA.  MMAs and copies
// complete on mbarriers.  Every wait is bounded in time; a give-up records
// PKV_DEVERR_TIMEOUT and raises a CTA-wide abort flag that every other wait
// also polls; then each role waits (bounded) for what it has in flight
// (MMAs, copies), tensor memory is freed and the CTA returns.
//
// Sizes: QT = 2 (256 rows): 192 KB of shared memory, 512 TMEM columns, one
// CTA per SM.  QT = 1: 96 KB, 256 columns, two CTAs per SM.  Either way the
// CTAs an SM can hold never ask for more than its 512 columns, so an
// allocation never waits on another CTA of this kernel.
#pragma once
#include "attention_fp8_tc.cuh"

namespace pkv {

namespace tc {

// Instruction descriptor of kind::f16: T x T -> F32, M = 128, N = n;
// b_mn: B read MN-major.  T = bf16 (format 1) or f16 (format 0).
template <typename T>
__host__ __device__ constexpr uint32_t idesc_f16_m128(uint32_t n, bool b_mn) {
    return (1u << 4)                                             // D format F32
           | ((std::is_same<T, __half>::value ? 0u : 1u) << 7)   // A format
           | ((std::is_same<T, __half>::value ? 0u : 1u) << 10)  // B format
           | (0u << 15)                                          // A K-major
           | ((b_mn ? 1u : 0u) << 16)                            // B major
           | ((n >> 3) << 17)                                    // N / 8
           | ((128u >> 4) << 24);                                // M / 16
}

// D (+)= A B, A and B from shared memory.
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

// D (+)= A B, A from tensor memory (lane = row, two 16-bit elements per
// 32-bit column), B from shared memory.
__device__ __forceinline__ void mma_f16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                               bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        :
        : "r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate ? 1u : 0u)
        : "memory");
}

#define PKV_TO8(b)                                                                                            \
    "=r"(r[b]), "=r"(r[b + 1]), "=r"(r[b + 2]), "=r"(r[b + 3]), "=r"(r[b + 4]), "=r"(r[b + 5]), "=r"(r[b + 6]), \
        "=r"(r[b + 7])
#define PKV_TI8(b) \
    "r"(v[b]), "r"(v[b + 1]), "r"(v[b + 2]), "r"(v[b + 3]), "r"(v[b + 4]), "r"(v[b + 5]), "r"(v[b + 6]), "r"(v[b + 7])

// Columns c .. c+31 (c+63) of this warp's 32 lanes (thread i of the warp: lane
// base + i); the values are complete when the call returns (the wait is in
// the same asm statement).
__device__ __forceinline__ void ld_x32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "{\n\ttcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;\n\t}"
        : PKV_TO8(0), PKV_TO8(8), PKV_TO8(16), PKV_TO8(24)
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void ld_x64(uint32_t taddr, uint32_t (&r)[64]) {
    asm volatile(
        "{\n\ttcgen05.ld.sync.aligned.32x32b.x64.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, "
        "%35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, "
        "%56, %57, %58, %59, %60, %61, %62, %63}, [%64];\n\t"
        "tcgen05.wait::ld.sync.aligned;\n\t}"
        : PKV_TO8(0), PKV_TO8(8), PKV_TO8(16), PKV_TO8(24), PKV_TO8(32), PKV_TO8(40), PKV_TO8(48), PKV_TO8(56)
        : "r"(taddr)
        : "memory");
}

// Store 32 columns of this warp's lanes; written when the call returns.
__device__ __forceinline__ void st_x32(uint32_t taddr, const uint32_t (&v)[32]) {
    asm volatile(
        "{\n\ttcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};\n\t"
        "tcgen05.wait::st.sync.aligned;\n\t}"
        :
        : "r"(taddr), PKV_TI8(0), PKV_TI8(8), PKV_TI8(16), PKV_TI8(24)
        : "memory");
}
#undef PKV_TO8
#undef PKV_TI8

}  // namespace tc

// Shared memory of the pass (offsets from a 1024-byte aligned base).
template <int QT, int KS, int VS>
struct PrefixTcCfg {
    static constexpr int kTok = 64;            // tokens per K / V tile
    static constexpr int kQBlk = 128 * 128;    // 128 query rows x 64 head-dim elements (16 KB)
    static constexpr int kHalf = kTok * 128;   // 64 token rows x 64 head-dim elements (8 KB)
    static constexpr int kTile = 2 * kHalf;    // one K or V tile, both head-dim halves
    static constexpr int kQOff = 0;            // Q tile q: blocks 2q, 2q+1
    static constexpr int kKOff = kQOff + QT * 2 * kQBlk;
    static constexpr int kVOff = kKOff + KS * kTile;
    static constexpr int kBarOff = kVOff + VS * kTile;
    // kfull[KS], kempty[KS], vfull[VS], vempty[VS]; per Q tile sfull[2],
    // pfull[2], obar, ofin; drain
    static constexpr int kBars = 2 * KS + 2 * VS + 6 * QT + 1;
    static constexpr int kTmemOff = kBarOff + 8 * kBars;
    static constexpr int kAbortOff = kTmemOff + 4;
    static constexpr int kSmemBytes = 1024 + kAbortOff + 4;
    static constexpr int kCols = 256 * QT;     // per Q tile: S / P buffers at 0 and 64, O at 128-255
    static constexpr int kWarps = 4 * QT + 3;  // softmax warpgroups, K copies, V copies, MMA
    static constexpr int kThreads = 32 * kWarps;
    static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
    static_assert(QT == 2 || 2 * (kSmemBytes + 1024) <= 228 * 1024, "two CTAs per SM at QT = 1");
    static_assert(3 * (kSmemBytes + 1024) > 228 * 1024, "at most two CTAs per SM (tensor-memory columns)");
    static_assert(QT == 1 || 2 * (kSmemBytes + 1024) > 228 * 1024, "one CTA per SM at QT = 2");
};

// A reference maximum moves only when a tile's maximum (log2 units) exceeds it
// by more than this, so softmax weights stay below 2^8.
constexpr float kPrefixRescaleLog2 = 8.f;

// Bounded wait that also gives up once another role of the CTA has raised
// the abort flag.
__device__ __forceinline__ bool mbar_wait_or_abort(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (global_ns() - t0 > kWaitLimitNs) {
            flag_error(8u /* PKV_DEVERR_TIMEOUT */);
            *abort_flag = 1;
            return false;
        }
    }
}

template <typename T, int QT, int KS, int VS>
__global__ void __launch_bounds__(PrefixTcCfg<QT, KS, VS>::kThreads, QT == 1 ? 2 : 1)
    prefix_attn_tc_kernel(const AttnParams p, const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV) {
    using C = PrefixTcCfg<QT, KS, VS>;
    constexpr int D = 128, TOK = C::kTok;
    constexpr int kWarpK = 4 * QT, kWarpV = 4 * QT + 1, kWarpM = 4 * QT + 2;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tile_r = blockIdx.x;  // 128*QT-row tile of the group
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
    const int row0 = tile_r * 128 * QT;
    if (row0 >= rows) return;  // CTA-uniform
    const int nq = min(QT, (rows - row0 + 127) / 128);  // Q tiles holding rows
    const int shared = p.group_shared[gi];
    if (shared <= 0 || shared % p.bs != 0 || shared > p.max_len || shared > p.max_shared) return;
    const int t0 = pp * p.P;
    if (t0 >= shared) return;
    const int t1 = min(shared, t0 + p.P);  // t1 - t0: a multiple of 16, as block sizes are
    const int n = (t1 - t0 + TOK - 1) / TOK;

    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t b_kfull = sbase + C::kBarOff, b_kempty = b_kfull + 8 * KS;
    const uint32_t b_vfull = b_kempty + 8 * KS, b_vempty = b_vfull + 8 * VS;
    const uint32_t b_q = b_vempty + 8 * VS;  // Q tile q at +48q: sfull[2], pfull[2], obar, ofin
    const uint32_t b_drain = b_q + 48 * QT;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kTmemOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kAbortOff);

    // softmax threads: this thread's query row
    const bool is_soft = warp < 4 * QT;
    const int q = warp >> 2;  // Q tile of a softmax thread
    const int t = tid & 127;  // its row in the tile = its TMEM lane
    const int r = row0 + q * 128 + t;
    const bool inrow = is_soft && r < rows;
    const int s_r = first + (inrow ? r / G : 0);
    const int h_r = g * G + (inrow ? r % G : 0);
    const bool live = inrow && p.member[s_r].x == gi + 1;

    // ---- set-up: tensor memory, barriers, Q
    if (warp == kWarpM) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"((uint32_t)C::kCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
    }
    if (tid == kWarpK * 32) {
        prefetch_tensor_map(&tmK);
        prefetch_tensor_map(&tmV);
        for (int i = 0; i < KS; ++i) {
            mbar_init(b_kfull + 8 * i, 1);
            mbar_init(b_kempty + 8 * i, 1);
        }
        for (int i = 0; i < VS; ++i) {
            mbar_init(b_vfull + 8 * i, 1);
            mbar_init(b_vempty + 8 * i, 1);
        }
        for (int i = 0; i < QT; ++i) {
            mbar_init(b_q + 48 * i, 1);
            mbar_init(b_q + 48 * i + 8, 1);
            mbar_init(b_q + 48 * i + 16, 128);  // every softmax thread of the Q tile
            mbar_init(b_q + 48 * i + 24, 128);
            mbar_init(b_q + 48 * i + 32, 1);
            mbar_init(b_q + 48 * i + 40, 1);
        }
        mbar_init(b_drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (is_soft && q < nq) {
        const uint4* qsrc = reinterpret_cast<const uint4*>(reinterpret_cast<const T*>(p.q) +
                                                             ((int64_t)s_r * p.Hq + h_r) * D);
        uint8_t* qrow = smem + C::kQOff + q * 2 * C::kQBlk + t * 128;
#pragma unroll
        for (int c = 0; c < 16; ++c) {  // 16-byte chunk c: block c / 8, chunk c % 8 of the row
            const uint4 v = live ? qsrc[c] : make_uint4(0u, 0u, 0u, 0u);
            *reinterpret_cast<uint4*>(qrow + (c >> 3) * C::kQBlk + (((c & 7) ^ (t & 7)) << 4)) = v;
        }
    }
    fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    int issued = 0;  // tiles whose copies this producer warp issued
    if (warp == kWarpK || warp == kWarpV) {
        // ---- copies: tile j into ring slot j % S, refilled once the MMAs
        // that read the slot's previous tile have completed
        const bool isv = warp == kWarpV;
        const int S = isv ? VS : KS;
        const uint32_t full = isv ? b_vfull : b_kfull, empty = isv ? b_vempty : b_kempty;
        const uint32_t ring = sbase + (isv ? C::kVOff : C::kKOff);
        const CUtensorMap* map = isv ? &tmV : &tmK;
        const int jb0 = t0 / p.bs;
        BlockWindow win;
        win.init(p.block_tables + (int64_t)first * p.maxB, jb0, (t1 - 1) / p.bs - jb0 + 1, lane);
        for (int j = 0; j < n; ++j) {
            const int slot = j % S;
            if (j >= S) {
                bool w = true;
                if (lane == 0) w = mbar_wait_or_abort(empty + 8 * slot, ((j / S) - 1) & 1, abort_flag);
                if (!__shfl_sync(0xffffffffu, w ? 1 : 0, 0)) break;
            }
            const int tt0 = t0 + j * TOK;
            const int nbox = min(TOK, t1 - tt0) / kTileTok;
            const uint32_t dst = ring + slot * C::kTile, bar = full + 8 * slot;
            if (lane == 0) mbar_arrive_expect_tx(bar, (uint32_t)(nbox * kTileTok * D * 2));
            for (int b = 0; b < nbox; ++b) {
                const int th = tt0 + b * kTileTok;
                const int blk = win.get(th / p.bs - jb0, lane, p.NB);
                if (lane == 0) {
                    const int row = (blk * p.Hkv + g) * p.bs + (th % p.bs);
                    tma_load_2d(dst + b * kTileTok * 128, map, 0, row, bar);
                    tma_load_2d(dst + C::kHalf + b * kTileTok * 128, map, 64, row, bar);
                }
            }
            issued = j + 1;
        }
    } else if (warp == kWarpM) {
        // ---- MMAs (lane 0): S of tile j+1 goes in before O += P V of tile j
        if (lane == 0) {
            constexpr uint32_t kIdS = tc::idesc_f16_m128<T>(64, false);
            constexpr uint32_t kIdO = tc::idesc_f16_m128<T>(128, true);
            auto issue_s = [&](int j) -> bool {
                const int slot = j % KS;
                if (!mbar_wait_or_abort(b_kfull + 8 * slot, (j / KS) & 1, abort_flag)) return false;
                tc::fence_after_sync();
                const uint32_t kb = sbase + C::kKOff + slot * C::kTile;
                for (int qq = 0; qq < nq; ++qq) {
                    const uint32_t qb = sbase + C::kQOff + qq * 2 * C::kQBlk;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        tc::mma_f16(tmem + qq * 256 + (j & 1) * 64,
                                    tc::smem_desc_sw128(qb + (kk >> 2) * C::kQBlk + (kk & 3) * 32, 16, 1024),
                                    tc::smem_desc_sw128(kb + (kk >> 2) * C::kHalf + (kk & 3) * 32, 16, 1024), kIdS,
                                    kk > 0);
                    tc::commit(b_q + 48 * qq + 8 * (j & 1));  // S of tile j ready
                }
                tc::commit(b_kempty + 8 * slot);  // K slot free
                return true;
            };
            bool ok = issue_s(0);
            for (int j = 0; ok && j < n; ++j) {
                if (j + 1 < n && !(ok = issue_s(j + 1))) break;
                const int slot = j % VS;
                if (!(ok = mbar_wait_or_abort(b_vfull + 8 * slot, (j / VS) & 1, abort_flag))) break;
                const int valid = min(TOK, t1 - (t0 + j * TOK));
                const uint32_t vb = sbase + C::kVOff + slot * C::kTile;
                for (int qq = 0; qq < nq; ++qq) {
                    if (!(ok = mbar_wait_or_abort(b_q + 48 * qq + 16 + 8 * (j & 1), (j >> 1) & 1, abort_flag))) break;
                    tc::fence_after_sync();
                    for (int kk = 0; kk < valid / 16; ++kk)
                        tc::mma_f16_tmem_a(tmem + qq * 256 + 128, tmem + qq * 256 + (j & 1) * 64 + kk * 8,
                                           tc::smem_desc_sw128(vb + kk * 16 * 128, C::kHalf, 1024), kIdO,
                                           j > 0 || kk > 0);
                    tc::commit(b_q + 48 * qq + 32);  // O products of tile j done
                }
                if (!ok) break;
                tc::commit(b_vempty + 8 * slot);  // V slot free
            }
            if (ok)
                for (int qq = 0; qq < nq; ++qq) tc::commit(b_q + 48 * qq + 40);  // O final
            // every MMA issued, and so every arrival it owes, has completed
            // before the CTA can leave (bounded)
            tc::commit(b_drain);
            mbar_wait(b_drain, 0);
        }
        __syncwarp();
    } else if (q < nq) {
        // ---- softmax of Q tile q: thread t owns row t (TMEM lane t)
        const uint32_t tq = tmem + ((uint32_t)((warp & 3) * 32) << 16) + q * 256;
        const uint32_t sfull = b_q + 48 * q, pfull = sfull + 16, obar = sfull + 32, ofin = sfull + 40;
        const float sl2 = p.scale_log2;
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < n; ++j) {
            const bool w = mbar_wait_or_abort(sfull + 8 * (j & 1), (j >> 1) & 1, abort_flag);
            if (!__all_sync(0xffffffffu, w)) {
                ok = false;
                break;
            }
            tc::fence_after_sync();
            uint32_t sr[64];
            tc::ld_x64(tq + (j & 1) * 64, sr);
            const int valid = min(TOK, t1 - (t0 + j * TOK));
            float x[64];
            float mt = -INFINITY;
#pragma unroll
            for (int k = 0; k < 64; ++k) {
                x[k] = __uint_as_float(sr[k]) * sl2;
                if (k < valid) mt = fmaxf(mt, x[k]);
            }
            const bool need = mt > m + kPrefixRescaleLog2;  // always on the first tile
            const float mn = need ? mt : m;
            const float alpha = ex2(m - mn);  // 1 when m stays; 0 on the first tile (m = -inf)
            uint32_t pw[32];
            float ls = 0.f;
#pragma unroll
            for (int k = 0; k < 64; k += 2) {
                const float p0 = k < valid ? ex2(x[k] - mn) : 0.f;
                const float p1 = k + 1 < valid ? ex2(x[k + 1] - mn) : 0.f;
                ls += p0 + p1;
                pw[k / 2] = Elt<T>::pack2(p0, p1);
            }
            if (j > 0 && __any_sync(0xffffffffu, need)) {
                // the previous tile's O products must have landed before O is rescaled
                const bool w2 = mbar_wait_or_abort(obar, (j - 1) & 1, abort_flag);
                if (!__all_sync(0xffffffffu, w2)) {
                    ok = false;
                    break;
                }
                tc::fence_after_sync();
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    tc::ld_x32(tq + 128 + c * 32, o);
#pragma unroll
                    for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
                    tc::st_x32(tq + 128 + c * 32, o);
                }
            }
            l = l * alpha + ls;
            m = mn;
            tc::st_x32(tq + (j & 1) * 64, pw);  // P over the scores it came from
            tc::fence_before_sync();
            mbar_arrive(pfull + 8 * (j & 1));
        }
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait_or_abort(ofin, 0, abort_flag));
        if (ok) {
            // ---- the row's partial: o (unnormalised, at reference maximum m), m, l
            tc::fence_after_sync();
            const int64_t idx = ((int64_t)s_r * p.Hq + h_r) * p.maxP + pp;
            float* dst = p.ws_o + idx * D;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                tc::ld_x32(tq + 128 + c * 32, o);
                if (live) {
#pragma unroll
                    for (int k = 0; k < 32; k += 4)
                        *reinterpret_cast<float4*>(dst + c * 32 + k) =
                            make_float4(__uint_as_float(o[k]), __uint_as_float(o[k + 1]), __uint_as_float(o[k + 2]),
                                        __uint_as_float(o[k + 3]));
                }
            }
            if (live) *reinterpret_cast<float2*>(p.ws_ml + idx * 2) = make_float2(m, l);
        }
    }

    // ---- teardown: after a give-up, the copies still in flight land first
    // (bounded); the MMA warp has drained its MMAs above
    __syncthreads();
    if (*abort_flag && (warp == kWarpK || warp == kWarpV) && lane == 0) {
        const int S = warp == kWarpV ? VS : KS;
        const uint32_t full = warp == kWarpV ? b_vfull : b_kfull;
        for (int j = max(0, issued - S); j < issued; ++j)  // the last tile issued into each slot
            mbar_wait(full + 8 * (j % S), (j / S) & 1);
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == kWarpM) {
        tc::fence_after_sync();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)C::kCols));
    }
}

}  // namespace pkv
