// Paged decode attention on tensor cores (mma.sync m16n8k16, fp32 accumulate).
//
// Two kernels share one per-warp core that streams a token range of one kv
// head through a shared-memory ring and attends 16 query rows to it:
//
//  * paged_attn_mma_kernel -- grouped-query attention: one warp per
//    (sequence, kv head, partition); its 16 rows are the G query heads of the
//    group (2 <= G <= 16, padded with zero rows), so every K/V byte serves G
//    queries.
//  * prefix_attn_mma_kernel -- sequences that share their first tokens (a
//    system prompt stored once: openeuler.csdn.net PagedAttention explainer
//    6.1; aiknowledge.cn "2.2 PagedAttention 与 KV Cache 分页管理" 2.2.3):
//    one warp per (group, 16 query rows, kv head, partition of the shared
//    tokens); its rows are (sequence, head) pairs of 16 different queries of
//    the group, all attending to the same shared blocks, so each shared K/V
//    tile is read once per 16 queries instead of once per query.  Results are
//    split-K partials merged with each sequence's own partitions by the
//    reduce kernel.
//
// Per 16-token tile (tokens of one block, found through the block table;
// explainer 4.2, aiknowledge.cn 2.2.3-2.2.4):
//   S = Q K^T   A = Q rows (registers, loaded once per unit), B = K^T from the
//               shared-memory tile via ldmatrix (a K row is a column of B).
//   online softmax on the accumulator fragments (each row is spread over the
//               4 lanes of a quad), log2 domain.
//   O += P V    P re-packed from the S accumulators into A fragments in
//               registers; B = V via ldmatrix.trans.
//
// Data movement: each stage is one 16-token tile of K and one of V, loaded by
// 2-D tensor TMA (box 64 elements x 16 rows) with 128-byte swizzle, so the 8
// rows one ldmatrix phase reads fall in 8 different bank groups.  The tensor
// maps view a pool as a (num_blocks*Hkv*block_size) x D matrix; row
// (block*Hkv + g)*block_size + offset holds a token's K (or V) for kv head g.
#pragma once
#include <type_traits>

#include "attention_common.cuh"

namespace pkv {

// Shared memory of one warp: STAGES stages of (K tile, V tile), 16-bit
// swizzled tiles as loaded by TMA.
template <typename T, int D, int WARPS, int STAGES>
struct MmaCfg {
    static constexpr int kHalfTile = kTileTok * 128;     // 16 rows x 64 16-bit elements (bytes)
    static constexpr int kTileBytes = kTileTok * D * 2;  // one K (or V) tile
    static constexpr int kStageBytes = 2 * kTileBytes;
    static constexpr int kWarpBytes = STAGES * kStageBytes;
    static constexpr int kDataBytes = WARPS * kWarpBytes;
    static constexpr int kSmemBytes = 1024 + kDataBytes + WARPS * STAGES * 8;  // + alignment slack
    static_assert(D % 64 == 0, "head_dim must be a multiple of 64");
};

// Attention state of one warp over 16 query rows.  Accumulator element e of
// output n-tile j is row gid (e < 2) or gid + 8 (e >= 2), column j*8 + 2*tig + (e & 1).
template <typename T, int D>
struct MmaAcc {
    static constexpr int KSTEPS = D / 16;
    static constexpr int NT_O = D / 8;
    uint32_t qa[KSTEPS][4];  // Q as A fragments
    float o[NT_O][4];
    float m_lo, m_hi, l_lo, l_hi;

    // Two Tq elements -> a T pair (converted through fp32 when the types differ).
    template <typename Tq>
    __device__ __forceinline__ static uint32_t pair(const Tq* p) {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
        if constexpr (std::is_same<Tq, T>::value) {
            return w;
        } else {
            float f[2];
            Elt<Tq>::widen2(w, f);
            return Elt<T>::pack2(f[0], f[1]);
        }
    }

    // Row pointers (nullptr = zero row).
    template <typename Tq>
    __device__ __forceinline__ void load_q(const Tq* row_lo, const Tq* row_hi, int tig) {
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
            const int c0 = kk * 16 + 2 * tig;
            qa[kk][0] = row_lo ? pair(row_lo + c0) : 0u;
            qa[kk][1] = row_hi ? pair(row_hi + c0) : 0u;
            qa[kk][2] = row_lo ? pair(row_lo + c0 + 8) : 0u;
            qa[kk][3] = row_hi ? pair(row_hi + c0 + 8) : 0u;
        }
#pragma unroll
        for (int j = 0; j < NT_O; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
        m_lo = m_hi = -INFINITY;
        l_lo = l_hi = 0.f;
    }
};

// Online-softmax step for one 16 x 16 score tile (log2 domain).  sacc holds
// the raw scores, element e of n-tile nt being token nt*8 + 2*tig + (e & 1) of
// row gid (e < 2) or gid + 8 (e >= 2); row gid sees the first seen_lo tokens,
// row gid + 8 the first seen_hi; scale_lo / scale_hi turn the raw scores of
// the two rows into the log2 domain.  Updates the running max and sum, rescales
// the output accumulators and returns the probabilities packed as the A
// fragments of the P V product.  HI = false: rows 8..15 are padding (at most
// 8 live rows), so their state is left alone and their probabilities are 0.
template <typename T, int D, bool HI = true>
__device__ __forceinline__ void mma_softmax(MmaAcc<T, D>& acc, float (&sacc)[2][4], int tig, int seen_lo,
                                            int seen_hi, float scale_lo, float scale_hi, uint32_t (&pa)[4]) {
    constexpr int NT_O = D / 8;
    constexpr int NE = HI ? 4 : 2;  // accumulator elements of live rows
    if (__all_sync(0xffffffffu, seen_lo >= kTileTok && (!HI || seen_hi >= kTileTok))) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < NE; ++e) sacc[nt][e] *= e < 2 ? scale_lo : scale_hi;
    } else {  // a partial tile or a causal limit inside it
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
            for (int e = 0; e < NE; ++e) {
                const int tok = nt * 8 + 2 * tig + (e & 1);
                sacc[nt][e] = tok < (e < 2 ? seen_lo : seen_hi) ? sacc[nt][e] * (e < 2 ? scale_lo : scale_hi)
                                                                : -INFINITY;
            }
        }
    }
    float mx_lo = fmaxf(fmaxf(sacc[0][0], sacc[0][1]), fmaxf(sacc[1][0], sacc[1][1]));
    float mx_hi = HI ? fmaxf(fmaxf(sacc[0][2], sacc[0][3]), fmaxf(sacc[1][2], sacc[1][3])) : 0.f;
#pragma unroll
    for (int off = 1; off < 4; off <<= 1) {
        mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, off));
        if (HI) mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, off));
    }
    const float mn_lo = fmaxf(acc.m_lo, mx_lo), mn_hi = HI ? fmaxf(acc.m_hi, mx_hi) : 0.f;
    // A row that has seen no token yet keeps m = -inf; exponentiate against 0
    // then, so that no -inf - -inf appears.
    const float b_lo = mn_lo == -INFINITY ? 0.f : mn_lo, b_hi = mn_hi == -INFINITY ? 0.f : mn_hi;
    const float a_lo = ex2(acc.m_lo - b_lo), a_hi = HI ? ex2(acc.m_hi - b_hi) : 1.f;
    acc.m_lo = mn_lo;
    if (HI) acc.m_hi = mn_hi;
    float ps_lo = 0.f, ps_hi = 0.f;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
        for (int e = 0; e < NE; ++e) {
            const float pr = ex2(sacc[nt][e] - (e < 2 ? b_lo : b_hi));
            sacc[nt][e] = pr;
            if (e < 2) ps_lo += pr;
            else ps_hi += pr;
        }
    }
    acc.l_lo = acc.l_lo * a_lo + ps_lo;
    if (HI) acc.l_hi = acc.l_hi * a_hi + ps_hi;
    // Once the running maxima settle, every factor is exactly 1 and the
    // multiplications change nothing: skip them when that holds warp-wide.
    if (!__all_sync(0xffffffffu, a_lo == 1.f && a_hi == 1.f)) {
#pragma unroll
        for (int j = 0; j < NT_O; ++j) {
            acc.o[j][0] *= a_lo;
            acc.o[j][1] *= a_lo;
            if (HI) {
                acc.o[j][2] *= a_hi;
                acc.o[j][3] *= a_hi;
            }
        }
    }
    pa[0] = Elt<T>::pack2(sacc[0][0], sacc[0][1]);
    pa[1] = HI ? Elt<T>::pack2(sacc[0][2], sacc[0][3]) : 0u;
    pa[2] = Elt<T>::pack2(sacc[1][0], sacc[1][1]);
    pa[3] = HI ? Elt<T>::pack2(sacc[1][2], sacc[1][3]) : 0u;
}

// Per-lane wait for stage st of tile i; on a timeout anywhere in the warp,
// drain the copies still in flight (tiles i+1 .. i+STAGES-1) and report false.
template <int STAGES>
__device__ __forceinline__ bool ring_wait(uint32_t bar0, int i, int ntiles) {
    const bool ok = mbar_wait(bar0 + 8 * (i % STAGES), (i / STAGES) & 1);
    if (__all_sync(0xffffffffu, ok)) return true;
    for (int k = i + 1; k < ntiles && k < i + STAGES; ++k) mbar_wait(bar0 + 8 * (k % STAGES), (k / STAGES) & 1);
    return false;
}

// Stream tokens [t_begin, t_end) of kv head g (block ids from bt_row) through
// this warp's ring and accumulate into acc.  Row gid sees only tokens below
// lim_lo, row gid+8 only tokens below lim_hi (causal chunks; pass t_end when
// every row sees the whole range).  Returns false if a wait on a copy timed
// out (the unit is then abandoned after draining its copies).
template <typename T, int D, int WARPS, int STAGES>
__device__ __forceinline__ bool mma_attend(const AttnParams& p, const CUtensorMap* tmK, const CUtensorMap* tmV,
                                           uint8_t* ring, uint32_t bar0, const int32_t* bt_row, int t_begin,
                                           int t_end, int g, int lane, MmaAcc<T, D>& acc, int lim_lo,
                                           int lim_hi) {
    using C = MmaCfg<T, D, WARPS, STAGES>;
    constexpr int KSTEPS = D / 16;
    const int tig = lane & 3;
    const int ntiles = (t_end - t_begin + kTileTok - 1) / kTileTok;
    const uint32_t ring_s = smem_u32(ring);

    const int jb0 = t_begin / p.bs;
    BlockWindow win;
    win.init(bt_row, jb0, (t_end - 1) / p.bs - jb0 + 1, lane);

    auto issue = [&](int i) {
        const int t0 = t_begin + i * kTileTok;
        const int blk = win.get(t0 / p.bs - jb0, lane, p.NB);
        if (lane == 0) {
            const int row = (blk * p.Hkv + g) * p.bs + (t0 % p.bs);
            const int st = i % STAGES;
            const uint32_t bar = bar0 + 8 * st;
            const uint32_t dst = ring_s + st * C::kStageBytes;
            fence_proxy_async();
            mbar_arrive_expect_tx(bar, C::kStageBytes);
#pragma unroll
            for (int hx = 0; hx < D / 64; ++hx) {
                tma_load_2d(dst + hx * C::kHalfTile, tmK, hx * 64, row, bar);
                tma_load_2d(dst + C::kTileBytes + hx * C::kHalfTile, tmV, hx * 64, row, bar);
            }
        }
    };

    const int npre = ntiles < STAGES ? ntiles : STAGES;
    for (int i = 0; i < npre; ++i) issue(i);

    // Per-lane ldmatrix row addresses.
    const int mi = lane >> 3, ri = lane & 7;
    const int k_tok = (mi >> 1) * 8 + ri;  // K: matrices (tok 0-7|8-15) x (d lo|hi)
    const int k_hi = mi & 1;
    const int v_tok = (mi & 1) * 8 + ri;   // V (trans): (tok lo|hi) x (d lo|hi)
    const int v_hi = mi >> 1;

    for (int i = 0; i < ntiles; ++i) {
        const int st = i % STAGES;
        if (!ring_wait<STAGES>(bar0, i, ntiles)) return false;
        const int valid = min(kTileTok, t_end - (t_begin + i * kTileTok));
        const int seen_lo = min(valid, lim_lo - (t_begin + i * kTileTok));  // tokens row gid sees
        const int seen_hi = min(valid, lim_hi - (t_begin + i * kTileTok));  // ... and row gid+8
        const uint32_t Ks = ring_s + st * C::kStageBytes;
        const uint32_t Vs = Ks + C::kTileBytes;
        uint8_t* vtile = ring + st * C::kStageBytes + C::kTileBytes;

        // S = Q K^T  (16 rows x 16 tokens as two n-tiles of 8 tokens)
        float sacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
            const int chunk = kk * 2 + k_hi;
            const uint32_t addr = Ks + (chunk >> 3) * C::kHalfTile + k_tok * 128 + (((chunk & 7) ^ (k_tok & 7)) << 4);
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4(addr, b0, b1, b2, b3);
            mma_16816<T>(sacc[0], acc.qa[kk], b0, b1);
            mma_16816<T>(sacc[1], acc.qa[kk], b2, b3);
        }
        uint32_t pa[4];
        mma_softmax(acc, sacc, tig, seen_lo, seen_hi, p.scale_log2, p.scale_log2, pa);

        // Rows past the context may hold anything (even NaN): zero them in V so
        // that 0-weights cannot turn into NaN inside the MMA.
        if (valid < kTileTok) {
            for (int idx = lane; idx < (kTileTok - valid) * (D / 8); idx += 32) {
                const int r = valid + idx / (D / 8);
                const int q16 = idx % (D / 8);  // 16-byte unit in the row (any order)
                *reinterpret_cast<uint4*>(vtile + (q16 >> 3) * C::kHalfTile + r * 128 + (q16 & 7) * 16) =
                    make_uint4(0u, 0u, 0u, 0u);
            }
            fence_proxy_async();  // these generic writes precede a later TMA refill
            __syncwarp();
        }

        // O += P V
#pragma unroll
        for (int jj = 0; jj < D / 16; ++jj) {
            const int chunk = jj * 2 + v_hi;
            const uint32_t addr = Vs + (chunk >> 3) * C::kHalfTile + v_tok * 128 + (((chunk & 7) ^ (v_tok & 7)) << 4);
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4_trans(addr, b0, b1, b2, b3);
            mma_16816<T>(acc.o[2 * jj], pa, b0, b1);
            mma_16816<T>(acc.o[2 * jj + 1], pa, b2, b3);
        }
        __syncwarp();
        if (i + STAGES < ntiles) issue(i + STAGES);
    }
#pragma unroll
    for (int off = 1; off < 4; off <<= 1) {
        acc.l_lo += __shfl_xor_sync(0xffffffffu, acc.l_lo, off);
        acc.l_hi += __shfl_xor_sync(0xffffffffu, acc.l_hi, off);
    }
    return true;
}

// Write one accumulator row, scaled by vs (the V code scale, 1 for 16-bit
// pools): the normalised output of type To (out_row != nullptr) or a split-K
// partial (o_row, ml).  hi selects rows gid+8.
template <typename To, typename T, int D>
__device__ __forceinline__ void mma_store_row(const MmaAcc<T, D>& acc, bool hi, int tig, To* out_row, float* o_row,
                                              float* ml, float vs) {
    constexpr int NT_O = D / 8;
    const int e0 = hi ? 2 : 0;
    const float l = hi ? acc.l_hi : acc.l_lo;
    if (out_row) {
        const float inv = vs / l;
#pragma unroll
        for (int j = 0; j < NT_O; ++j)
            *reinterpret_cast<uint32_t*>(out_row + j * 8 + 2 * tig) =
                Elt<To>::pack2(acc.o[j][e0] * inv, acc.o[j][e0 + 1] * inv);
    } else {
#pragma unroll
        for (int j = 0; j < NT_O; ++j)
            *reinterpret_cast<float2*>(o_row + j * 8 + 2 * tig) =
                make_float2(acc.o[j][e0] * vs, acc.o[j][e0 + 1] * vs);
        if (tig == 0) *reinterpret_cast<float2*>(ml) = make_float2(hi ? acc.m_hi : acc.m_lo, l);
    }
}

// One warp's ring: WARP_BYTES of stages at smem + warp * WARP_BYTES (smem
// 1024-byte aligned), its STAGES mbarriers after all warps' data.
template <int WARP_BYTES, int DATA_BYTES, int STAGES>
__device__ __forceinline__ uint8_t* ring_setup(uint8_t* smem_raw, int warp, int lane, uint32_t& bar0,
                                               const CUtensorMap* tmK, const CUtensorMap* tmV) {
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    bar0 = smem_u32(smem + DATA_BYTES + warp * STAGES * 8);
    if (lane == 0) {
        prefetch_tensor_map(tmK);
        prefetch_tensor_map(tmV);
        for (int i = 0; i < STAGES; ++i) mbar_init(bar0 + 8 * i, 1);
        fence_barrier_init();
    }
    __syncwarp();
    return smem + warp * WARP_BYTES;
}

template <typename T, int D, int WARPS, int STAGES>
__device__ __forceinline__ uint8_t* mma_setup_ring(uint8_t* smem_raw, int warp, int lane, uint32_t& bar0,
                                                   const CUtensorMap* tmK, const CUtensorMap* tmV) {
    using C = MmaCfg<T, D, WARPS, STAGES>;
    return ring_setup<C::kWarpBytes, C::kDataBytes, STAGES>(smem_raw, warp, lane, bar0, tmK, tmV);
}

// Grouped-query decode: grid (ceil(Hkv / WARPS), partitions, S).
template <typename T, int D, int WARPS, int STAGES>
__global__ void __launch_bounds__(WARPS * 32) paged_attn_mma_kernel(const AttnParams p,
                                                                    const __grid_constant__ CUtensorMap tmK,
                                                                    const __grid_constant__ CUtensorMap tmV) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g = blockIdx.x * WARPS + warp;  // kv head
    const int part = blockIdx.y;
    const int s = blockIdx.z;
    if (g >= p.Hkv) return;
    const int gid = lane >> 2, tig = lane & 3;
    const int G = p.G;
    const int h0 = g * G;

    const Unit u = resolve_unit(p, s, part, part == 0 && g == 0 && lane == 0);
    if (u.t_begin >= u.L) {
        if (part == 0 && u.L == 0) {  // empty context: zeros for the group's heads
            T* o = reinterpret_cast<T*>(p.out) + ((int64_t)s * p.Hq + h0) * D;
            for (int i = lane; i < G * D; i += 32) o[i] = T(0.f);
        }
        return;
    }
    uint32_t bar0;
    uint8_t* ring = mma_setup_ring<T, D, WARPS, STAGES>(smem_raw, warp, lane, bar0, &tmK, &tmV);

    const T* qb = reinterpret_cast<const T*>(p.q) + ((int64_t)s * p.Hq + h0) * D;
    MmaAcc<T, D> acc;
    acc.load_q(gid < G ? qb + gid * D : nullptr, gid + 8 < G ? qb + (gid + 8) * D : nullptr, tig);
    if (!mma_attend<T, D, WARPS, STAGES>(p, &tmK, &tmV, ring, bar0, p.block_tables + (int64_t)s * p.maxB,
                                         u.t_begin, u.t_end, g, lane, acc, u.t_end, u.t_end))
        return;

#pragma unroll
    for (int hi = 0; hi < 2; ++hi) {
        const int r = gid + 8 * hi;
        if (r >= G) continue;
        const int64_t row = (int64_t)s * p.Hq + h0 + r;
        if (u.direct) {
            mma_store_row<T, T, D>(acc, hi, tig, reinterpret_cast<T*>(p.out) + row * D, nullptr, nullptr, 1.f);
        } else {
            const int64_t idx = row * p.maxP + u.slot;
            mma_store_row<T, T, D>(acc, hi, tig, (T*)nullptr, p.ws_o + idx * D, p.ws_ml + idx * 2, 1.f);
        }
    }
}

// Shared-prefix pass: grid (row tiles, prefix partitions, groups * Hkv).  Row r
// of group i is (sequence group_first[i] + r / G, query head g*G + r % G).
// The WARPS warps of a CTA split the partition's tokens of one 16-row tile
// (so each warp's chain of dependent tile loads is short), then merge their
// (m, l, o) in shared memory into the single partial of that partition.
template <typename T, int D, int WARPS, int STAGES>
__global__ void __launch_bounds__(WARPS * 32) prefix_attn_mma_kernel(const AttnParams p,
                                                                     const __grid_constant__ CUtensorMap tmK,
                                                                     const __grid_constant__ CUtensorMap tmV) {
    using C = MmaCfg<T, D, WARPS, STAGES>;
    constexpr int NT_O = D / 8;
    static_assert(WARPS * 16 * (D + 2) * 4 <= C::kDataBytes, "merge buffer must fit in the ring");
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int tile = blockIdx.x;
    const int pp = blockIdx.y;  // partition of the shared tokens
    const int gi = blockIdx.z / p.Hkv;
    const int g = blockIdx.z - gi * p.Hkv;
    const int gid = lane >> 2, tig = lane & 3;
    const int G = p.G;

    int first = p.group_first[gi], last = p.group_first[gi + 1];
    first = max(0, min(first, p.S));
    last = max(first, min(last, p.S));
    if (last - first > p.max_group_size) {
        if (tile == 0 && pp == 0 && g == 0 && threadIdx.x == 0) flag_error(16u /* PKV_DEVERR_GROUP */);
        last = first + p.max_group_size;  // members past the grid get no prefix partials
    }
    const int rows = (last - first) * G;
    if (tile * 16 >= rows) return;
    const int shared = p.group_shared[gi];
    if (shared <= 0 || shared % p.bs != 0 || shared > p.max_len || shared > p.max_shared)
        return;  // reported by the decode kernels
    const int t0 = pp * p.P;
    if (t0 >= shared) return;
    const int t1 = min(shared, t0 + p.P);
    // This warp's share of [t0, t1), in whole 16-token tiles.
    const int per = ((t1 - t0 + WARPS * kTileTok - 1) / (WARPS * kTileTok)) * kTileTok;
    const int w0 = min(t1, t0 + warp * per), w1 = min(t1, w0 + per);

    // Query rows of this lane (gid, gid+8).  Only rows whose sequence takes
    // this group's prefix result (decided once per call, see
    // group_members_kernel) are attended and written.
    int rs[2], rh[2];
    bool use[2];
#pragma unroll
    for (int hi = 0; hi < 2; ++hi) {
        const int r = tile * 16 + gid + 8 * hi;
        use[hi] = r < rows && p.member[first + r / G].x == gi + 1;
        rs[hi] = first + (use[hi] ? r / G : 0);
        rh[hi] = g * G + (use[hi] ? r % G : 0);
    }
    uint32_t bar0;
    uint8_t* ring = mma_setup_ring<T, D, WARPS, STAGES>(smem_raw, warp, lane, bar0, &tmK, &tmV);
    const T* q = reinterpret_cast<const T*>(p.q);
    MmaAcc<T, D> acc;
    acc.load_q(use[0] ? q + ((int64_t)rs[0] * p.Hq + rh[0]) * D : nullptr,
               use[1] ? q + ((int64_t)rs[1] * p.Hq + rh[1]) * D : nullptr, tig);
    bool ok = true;
    if (w0 < w1)
        ok = mma_attend<T, D, WARPS, STAGES>(p, &tmK, &tmV, ring, bar0, p.block_tables + (int64_t)first * p.maxB,
                                             w0, w1, g, lane, acc, w1, w1);
    const int all_ok = __syncthreads_and(ok ? 1 : 0);  // every warp is done with its ring

    // Merge buffer (reuses the rings): o [WARPS][16][D], then m, l [WARPS][16].
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* so = reinterpret_cast<float*>(base);
    float* sm = so + WARPS * 16 * D;
    float* sl = sm + WARPS * 16;
#pragma unroll
    for (int j = 0; j < NT_O; ++j) {
        const int col = j * 8 + 2 * tig;
        *reinterpret_cast<float2*>(so + (warp * 16 + gid) * D + col) = make_float2(acc.o[j][0], acc.o[j][1]);
        *reinterpret_cast<float2*>(so + (warp * 16 + gid + 8) * D + col) = make_float2(acc.o[j][2], acc.o[j][3]);
    }
    if (tig == 0) {
        sm[warp * 16 + gid] = acc.m_lo;
        sm[warp * 16 + gid + 8] = acc.m_hi;
        sl[warp * 16 + gid] = acc.l_lo;
        sl[warp * 16 + gid + 8] = acc.l_hi;
    }
    __syncthreads();
    if (!all_ok) return;
    // Thread t merges row t / (WARPS*2) ... : 16 rows x D columns over the CTA.
    constexpr int kThreads = WARPS * 32;
    constexpr int kPerRow = kThreads / 16;   // threads per row
    constexpr int kCols = D / kPerRow;       // columns per thread
    static_assert(kCols % 4 == 0, "float4 columns");
    const int r = threadIdx.x / kPerRow;
    const int c0 = (threadIdx.x % kPerRow) * kCols;
    const int rr = tile * 16 + r;
    if (rr >= rows) return;
    const int s_r = first + rr / G, h_r = g * G + rr % G;
    if (p.member[s_r].x != gi + 1) return;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) M = fmaxf(M, sm[w * 16 + r]);
    float f[WARPS], lsum = 0.f;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) {
        f[w] = ex2(sm[w * 16 + r] - M);  // 0 for a warp that saw no token
        lsum += f[w] * sl[w * 16 + r];
    }
    const int64_t idx = ((int64_t)s_r * p.Hq + h_r) * p.maxP + pp;
    float* dst = p.ws_o + idx * D + c0;
#pragma unroll
    for (int cc = 0; cc < kCols; cc += 4) {
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w = 0; w < WARPS; ++w) {
            const float4 v = *reinterpret_cast<const float4*>(so + (w * 16 + r) * D + c0 + cc);
            a.x += f[w] * v.x;
            a.y += f[w] * v.y;
            a.z += f[w] * v.z;
            a.w += f[w] * v.w;
        }
        *reinterpret_cast<float4*>(dst + cc) = a;
    }
    if (c0 == 0) *reinterpret_cast<float2*>(p.ws_ml + idx * 2) = make_float2(M, lsum);
}

// Causal chunk of new tokens per sequence (speculative verification, chunked
// prefill): grid (ceil(Hkv / WARPS), row tiles * partitions, S).  The rows of
// sequence s for kv head g are (new token i, query head g*G + r) flattened as
// i*G + r; row i sits at position L - n + i and sees tokens 0 .. L - n + i
// (each token attends to itself and what precedes it: openeuler.csdn.net
// PagedAttention explainer 2.1-2.2).  16 rows per warp -- for multi-head
// attention 16 new tokens of one head, a real contraction over shared K/V.
template <typename T, int D, int WARPS, int STAGES>
__global__ void __launch_bounds__(WARPS * 32, 3) chunk_attn_mma_kernel(const AttnParams p, const ChunkParams c,
                                                                    const __grid_constant__ CUtensorMap tmK,
                                                                    const __grid_constant__ CUtensorMap tmV) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g = blockIdx.x * WARPS + warp;  // kv head
    const int part = blockIdx.y % c.nparts;
    const int tile = blockIdx.y / c.nparts;
    const int s = blockIdx.z;
    if (g >= p.Hkv) return;
    const int gid = lane >> 2, tig = lane & 3;
    const int G = p.G;
    const bool report = part == 0 && tile == 0 && g == 0 && lane == 0;

    const int L = load_context_len(p, s, report);
    const int q0 = c.query_start[s], q1 = c.query_start[s + 1];
    if (q0 < 0 || q1 < q0 || q1 > c.T || q1 - q0 > L || q1 - q0 > c.max_query_len) {
        if (report) flag_error(4u /* PKV_DEVERR_CONTEXT */);
        return;
    }
    const int n = q1 - q0;
    const int rows = n * G;
    if (tile * 16 >= rows) return;
    const int last_row = min(rows - 1, tile * 16 + 15);
    const int t_begin = part * p.P;
    const int t_end = min(min(L, t_begin + p.P), L - n + last_row / G + 1);
    if (t_begin >= t_end) return;

    int ri[2], rh[2], lim[2];
    bool use[2];
#pragma unroll
    for (int hi = 0; hi < 2; ++hi) {
        const int r = tile * 16 + gid + 8 * hi;
        use[hi] = r < rows;
        ri[hi] = use[hi] ? r / G : 0;
        rh[hi] = g * G + (use[hi] ? r % G : 0);
        lim[hi] = use[hi] ? L - n + ri[hi] + 1 : 0;  // tokens this row sees
    }
    uint32_t bar0;
    uint8_t* ring = mma_setup_ring<T, D, WARPS, STAGES>(smem_raw, warp, lane, bar0, &tmK, &tmV);
    const T* q = reinterpret_cast<const T*>(p.q);
    MmaAcc<T, D> acc;
    acc.load_q(use[0] ? q + ((int64_t)(q0 + ri[0]) * p.Hq + rh[0]) * D : nullptr,
               use[1] ? q + ((int64_t)(q0 + ri[1]) * p.Hq + rh[1]) * D : nullptr, tig);
    if (!mma_attend<T, D, WARPS, STAGES>(p, &tmK, &tmV, ring, bar0, p.block_tables + (int64_t)s * p.maxB, t_begin,
                                         t_end, g, lane, acc, lim[0], lim[1]))
        return;
    const bool direct = (L + p.P - 1) / p.P == 1;  // every row of the sequence has one partition
#pragma unroll
    for (int hi = 0; hi < 2; ++hi) {
        if (!use[hi] || lim[hi] <= t_begin) continue;  // no token of this row in the partition
        const int64_t row = (int64_t)(q0 + ri[hi]) * p.Hq + rh[hi];
        if (direct) {
            mma_store_row<T, T, D>(acc, hi, tig, reinterpret_cast<T*>(p.out) + row * D, nullptr, nullptr, p.v_scale);
        } else {
            const int64_t idx = row * p.maxP + part;
            mma_store_row<T, T, D>(acc, hi, tig, (T*)nullptr, p.ws_o + idx * D, p.ws_ml + idx * 2, p.v_scale);
        }
    }
}

}  // namespace pkv
