// Grouped-query paged decode over FP8 E4M3 pools on the tensor cores.
//
// Same unit of work as paged_attn_mma_kernel: one warp per (sequence, kv
// head, partition), the G query heads of the group being the 16 MMA rows
// (padded with zero rows), tokens found through the block table
// (openeuler.csdn.net PagedAttention explainer 4.2; aiknowledge.cn "2.2
// PagedAttention 与 KV Cache 分页管理" 2.2.3-2.2.4).  The K and V tiles stay in
// shared memory as E4M3 codes; each lane widens only the codes its own MMA
// fragments need, straight into registers.  Every E4M3 value is an FP16
// value, so the widening is exact and the MMA runs in FP16 with fp32
// accumulation; the per-pool scales fold into the softmax scale (K) and the
// final normalisation (V).
//
// Fragment layouts (mma.m16n8k16; lane = 4 * gid + tig).  A dot product may
// take its terms in any order, so each product's contraction index is
// permuted to make every lane's codes contiguous in the tile:
//  * S = Q K^T.  K-step kk, lane tig: the logical k indices {2tig, 2tig+1,
//    2tig+8, 2tig+9} are head-dim elements tig*D/4 + 4kk + {0, 1, 2, 3}.  A
//    lane reads D/4 consecutive codes of token nt*8 + gid (n-tile nt), and
//    the Q fragments follow the same map.
//  * O += P V.  The contraction runs over the tokens in the order of the S
//    columns (lane tig holds tokens 2tig, 2tig+1, 8+2tig, 9+2tig).  Output
//    n-tile j, column n is head-dim element n*D/8 + j, so a lane reads D/8
//    consecutive codes of each of its four tokens and pairs the codes of two
//    tokens with one byte permute per four columns.
//
// Tiles arrive by 2-D tensor TMA as 16 tokens x D codes.  D = 128: 128-byte
// rows with the 128-byte swizzle (16-byte chunk c of row r lands at chunk
// c ^ (r & 7)), under which the K reads (two chunks per lane: 2tig, 2tig+1)
// and the V reads (one chunk per lane: gid) of each quarter warp hit eight
// different chunk positions.  D = 64: 64-byte rows, no swizzle.
#pragma once
#include "attention_mma.cuh"

namespace pkv {

template <int D, int WARPS, int STAGES>
struct Fp8Cfg {
    static constexpr int kTileBytes = kTileTok * D;  // one K (or V) tile of codes
    static constexpr int kStageBytes = 2 * kTileBytes;
    static constexpr int kWarpBytes = STAGES * kStageBytes;
    static constexpr int kDataBytes = WARPS * kWarpBytes;
    static constexpr int kSmemBytes = 1024 + kDataBytes + WARPS * STAGES * 8;  // + alignment slack
    static constexpr bool kSwizzle = D == 128;
    static_assert(D == 64 || D == 128, "head_dim must be 64 or 128");
    static_assert(kTileBytes % 1024 == 0, "swizzled tiles must start on 1024-byte boundaries");
};

// Byte offset of the 16-byte chunk c of tile row r.
template <int D>
__device__ __forceinline__ int fp8_chunk(int r, int c) {
    if constexpr (D == 128) return r * 128 + ((c ^ (r & 7)) << 4);
    else return r * D + (c << 4);
}

// V rows past the context (the end of a partial tile) may hold any code, NaN
// included, and a zero weight times NaN would poison the sum: clear them in
// the stage before reading it (whole rows, so the swizzle does not matter).
template <int D>
__device__ __forceinline__ void zero_tail_rows(uint8_t* vt, int valid, int lane) {
    if (valid >= kTileTok) return;
    for (int idx = lane; idx < (kTileTok - valid) * (D / 16); idx += 32) {
        const int r = valid + idx / (D / 16);
        *reinterpret_cast<uint4*>(vt + r * D + (idx % (D / 16)) * 16) = make_uint4(0u, 0u, 0u, 0u);
    }
    fence_proxy_async();  // these generic writes precede the stage's next TMA refill
    __syncwarp();
}

// HI: more than 8 heads per group (rows 8..15 of the MMA are live).
template <int D, int WARPS, int STAGES, typename To, bool HI>
__global__ void __launch_bounds__(WARPS * 32, 3) paged_attn_fp8_kernel(const AttnParams p,
                                                                       const __grid_constant__ CUtensorMap tmK,
                                                                       const __grid_constant__ CUtensorMap tmV) {
    using C = Fp8Cfg<D, WARPS, STAGES>;
    constexpr int KSTEPS = D / 16;
    constexpr int NT_O = D / 8;
    constexpr int KW = KSTEPS;  // 32-bit words of K codes per lane and n-tile (D/4 codes)
    constexpr int VW = NT_O / 4;  // 32-bit words of V codes per lane and token (D/8 codes)
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
            To* o = reinterpret_cast<To*>(p.out) + ((int64_t)s * p.Hq + h0) * D;
            for (int i = lane; i < G * D; i += 32) o[i] = To(0.f);
        }
        return;
    }
    uint32_t bar0;
    uint8_t* ring = ring_setup<C::kWarpBytes, C::kDataBytes, STAGES>(smem_raw, warp, lane, bar0, &tmK, &tmV);
    const uint32_t ring_s = smem_u32(ring);

    // Q rows gid and gid + 8 as A fragments under the permuted contraction.
    MmaAcc<__half, D> acc;
    {
        const To* qb = reinterpret_cast<const To*>(p.q) + ((int64_t)s * p.Hq + h0) * D;
        const To* row_lo = gid < G ? qb + gid * D + tig * (D / 4) : nullptr;
        const To* row_hi = gid + 8 < G ? qb + (gid + 8) * D + tig * (D / 4) : nullptr;
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
            acc.qa[kk][0] = row_lo ? MmaAcc<__half, D>::pair(row_lo + 4 * kk) : 0u;
            acc.qa[kk][1] = row_hi ? MmaAcc<__half, D>::pair(row_hi + 4 * kk) : 0u;
            acc.qa[kk][2] = row_lo ? MmaAcc<__half, D>::pair(row_lo + 4 * kk + 2) : 0u;
            acc.qa[kk][3] = row_hi ? MmaAcc<__half, D>::pair(row_hi + 4 * kk + 2) : 0u;
        }
#pragma unroll
        for (int j = 0; j < NT_O; ++j) acc.o[j][0] = acc.o[j][1] = acc.o[j][2] = acc.o[j][3] = 0.f;
        acc.m_lo = acc.m_hi = -INFINITY;
        acc.l_lo = acc.l_hi = 0.f;
    }

    const int t_begin = u.t_begin, t_end = u.t_end;
    const int ntiles = (t_end - t_begin + kTileTok - 1) / kTileTok;
    const int32_t* bt_row = p.block_tables + (int64_t)s * p.maxB;
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
            tma_load_2d(dst, &tmK, 0, row, bar);
            tma_load_2d(dst + C::kTileBytes, &tmV, 0, row, bar);
        }
    };
    const int npre = ntiles < STAGES ? ntiles : STAGES;
    for (int i = 0; i < npre; ++i) issue(i);

    // This lane's tokens for the P V contraction, in S-column order.
    const int vtok[4] = {2 * tig, 2 * tig + 1, 8 + 2 * tig, 9 + 2 * tig};

    for (int i = 0; i < ntiles; ++i) {
        const int st = i % STAGES;
        if (!ring_wait<STAGES>(bar0, i, ntiles)) return;
        const int valid = min(kTileTok, t_end - (t_begin + i * kTileTok));
        const uint8_t* kt = ring + st * C::kStageBytes;
        const uint8_t* vt = kt + C::kTileBytes;

        // Codes of this lane's fragments, then the stage goes back to TMA.
        uint32_t kw[2][KW];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
            for (int c = 0; c < KW / 4; ++c) {
                const uint4 w = *reinterpret_cast<const uint4*>(kt + fp8_chunk<D>(nt * 8 + gid, tig * (KW / 4) + c));
                kw[nt][4 * c] = w.x;
                kw[nt][4 * c + 1] = w.y;
                kw[nt][4 * c + 2] = w.z;
                kw[nt][4 * c + 3] = w.w;
            }
        }
        zero_tail_rows<D>(const_cast<uint8_t*>(vt), valid, lane);
        uint32_t vw[4][VW];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            if constexpr (VW == 4) {
                const uint4 w = *reinterpret_cast<const uint4*>(vt + fp8_chunk<D>(vtok[t], gid));
                vw[t][0] = w.x;
                vw[t][1] = w.y;
                vw[t][2] = w.z;
                vw[t][3] = w.w;
            } else {
                const uint2 w = *reinterpret_cast<const uint2*>(vt + vtok[t] * D + gid * 8);
                vw[t][0] = w.x;
                vw[t][1] = w.y;
            }
        }
        __syncwarp();
        if (i + STAGES < ntiles) issue(i + STAGES);

        // S = Q K^T
        float sacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                uint32_t b0, b1;
                e4m3x4_to_f16x2x2(kw[nt][kk], b0, b1);
                mma_16816<__half>(sacc[nt], acc.qa[kk], b0, b1);
            }
        }
        uint32_t pa[4];
        mma_softmax<__half, D, HI>(acc, sacc, tig, valid, valid, p.scale_log2, p.scale_log2, pa);

        // O += P V
#pragma unroll
        for (int w = 0; w < VW; ++w) {
            // Bytes [x0, y0, x1, y1] and [x2, y2, x3, y3] of tokens x, y.
            const uint32_t lo0 = __byte_perm(vw[0][w], vw[1][w], 0x5140);
            const uint32_t hi0 = __byte_perm(vw[0][w], vw[1][w], 0x7362);
            const uint32_t lo1 = __byte_perm(vw[2][w], vw[3][w], 0x5140);
            const uint32_t hi1 = __byte_perm(vw[2][w], vw[3][w], 0x7362);
            uint32_t l0a, l0b, l1a, l1b, h0a, h0b, h1a, h1b;
            e4m3x4_to_f16x2x2(lo0, l0a, l0b);
            e4m3x4_to_f16x2x2(lo1, l1a, l1b);
            e4m3x4_to_f16x2x2(hi0, h0a, h0b);
            e4m3x4_to_f16x2x2(hi1, h1a, h1b);
            mma_16816<__half>(acc.o[4 * w], pa, l0a, l1a);
            mma_16816<__half>(acc.o[4 * w + 1], pa, l0b, l1b);
            mma_16816<__half>(acc.o[4 * w + 2], pa, h0a, h1a);
            mma_16816<__half>(acc.o[4 * w + 3], pa, h0b, h1b);
        }
    }
#pragma unroll
    for (int off = 1; off < 4; off <<= 1) {
        acc.l_lo += __shfl_xor_sync(0xffffffffu, acc.l_lo, off);
        acc.l_hi += __shfl_xor_sync(0xffffffffu, acc.l_hi, off);
    }

    // Lane (gid, tig) holds, for row gid (+8), the columns (2tig + e) * D/8 + j
    // (e = 0, 1; j = 0 .. D/8-1): two runs of D/8 consecutive elements.
#pragma unroll
    for (int hi = 0; hi < 2; ++hi) {
        const int r = gid + 8 * hi;
        if (r >= G) continue;
        const int64_t row = (int64_t)s * p.Hq + h0 + r;
        const int e0 = hi ? 2 : 0;
        const float l = hi ? acc.l_hi : acc.l_lo;
        if (u.direct) {
            const float inv = p.v_scale / l;
            To* out = reinterpret_cast<To*>(p.out) + row * D;
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                uint32_t h[NT_O / 2];
#pragma unroll
                for (int j = 0; j < NT_O; j += 2)
                    h[j / 2] = Elt<To>::pack2(acc.o[j][e0 + e] * inv, acc.o[j + 1][e0 + e] * inv);
                uint4* dst = reinterpret_cast<uint4*>(out + (2 * tig + e) * NT_O);
#pragma unroll
                for (int v = 0; v < NT_O / 8; ++v) dst[v] = make_uint4(h[4 * v], h[4 * v + 1], h[4 * v + 2], h[4 * v + 3]);
            }
        } else {
            const int64_t idx = row * p.maxP + u.slot;
            float* o_row = p.ws_o + idx * D;
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                float4* dst = reinterpret_cast<float4*>(o_row + (2 * tig + e) * NT_O);
#pragma unroll
                for (int v = 0; v < NT_O / 4; ++v)
                    dst[v] = make_float4(acc.o[4 * v][e0 + e] * p.v_scale, acc.o[4 * v + 1][e0 + e] * p.v_scale,
                                         acc.o[4 * v + 2][e0 + e] * p.v_scale, acc.o[4 * v + 3][e0 + e] * p.v_scale);
            }
            if (tig == 0) *reinterpret_cast<float2*>(p.ws_ml + idx * 2) = make_float2(hi ? acc.m_hi : acc.m_lo, l);
        }
    }
}

// Per-head decode over FP8 pools (multi-head attention: one query head per
// kv head, so no two queries share a K/V byte).  One warp per (sequence,
// query head, partition).  The tokens are the MMA rows and the query is the
// single live column of an n8 operand:
//  * S^T = K q^T.  A = the K tile (16 tokens x 16 head-dim elements per
//    k-step, rows gid and gid+8 per lane, the same permuted contraction as
//    above); B column 0 = q, held by the lanes with gid = 0, other columns 0.
//    The score of token gid (gid + 8) lands in the lane (gid, tig = 0).
//  * O^T += V^T p^T.  A = V^T: m-tile mt, row r is head-dim element
//    gid*D/8 + 2mt (r = gid) or gid*D/8 + 2mt + 1 (r = gid + 8); B column 0 =
//    p, held by the gid = 0 lanes.  A dot product may take its terms in any
//    order, so the contraction pairs up tokens j and j + 8, whose scores both
//    sit in lane (j, 0): that lane packs their two probabilities once, and
//    lane (0, tig) gathers the packs of lanes (2tig, 0) and (2tig+1, 0) with
//    two shuffles as its contraction indices (2tig, 2tig+1) and (2tig+8,
//    2tig+9).  The A operand follows: lane tig reads D/8 consecutive codes of
//    tokens 2tig, 2tig+8, 2tig+1, 2tig+9 and pairs the codes of two tokens
//    with one byte permute per four columns.  The lane (gid, tig = 0) ends
//    with output elements gid*D/8 .. gid*D/8 + D/8 - 1.
// Half the MMAs of the grouped layout (8 + 8 per 16 tokens at D = 128) and a
// quarter of the CUDA-core instructions of widening every code to fp32.
//
// TT tokens per pipeline stage (16 or 32): a 32-token stage is two 16-token
// tiles (each found through the block table on its own, so any block_size
// works) under one barrier, one softmax step and one loop iteration, which
// halves the fixed cost per token of everything but the widening and the
// MMAs.
template <int D, int TT>
struct Fp8HeadCfg {
    static constexpr int kHalves = TT / kTileTok;
    static constexpr int kTileBytes = kTileTok * D;           // one 16-token K (or V) tile of codes
    static constexpr int kStageBytes = 2 * kHalves * kTileBytes;  // K tiles, then V tiles
    static_assert(TT == 16 || TT == 32, "16 or 32 tokens per stage");
};

// LATE_V: the V codes are read from the stage after the softmax (the stage
// goes back to TMA then) instead of with the K codes, so the K and V codes
// are never held in registers at the same time.
template <int D, int WARPS, int STAGES, typename To, int TT = kTileTok, int MINB = 4, bool LATE_V = false>
__global__ void __launch_bounds__(WARPS * 32, MINB) paged_attn_fp8_head_kernel(const AttnParams p,
                                                                               const __grid_constant__ CUtensorMap tmK,
                                                                               const __grid_constant__ CUtensorMap tmV) {
    using C = Fp8HeadCfg<D, TT>;
    using H = MmaAcc<__half, D>;
    constexpr int HV = C::kHalves;
    constexpr int KSTEPS = D / 16;  // S^T k-steps; also 32-bit words of K codes per lane and row
    constexpr int NMT = D / 16;     // O^T m-tiles
    constexpr int VW = D / 32;      // 32-bit words of V codes per lane and token (D/8 codes)
    constexpr int SPAN = D / 8;     // output elements per lane with tig = 0
    constexpr int kWarpBytes = STAGES * C::kStageBytes;
    constexpr int kDataBytes = WARPS * kWarpBytes;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int h = blockIdx.x * WARPS + warp;  // query head
    int part = blockIdx.y;
    int s = blockIdx.z;
    if (p.lpt) {
        const int2 unit = lpt_unit_cta(p, blockIdx.z * gridDim.y + blockIdx.y);
        if (unit.x < 0) return;
        s = unit.x;
        part = unit.y;
    }
    if (h >= p.Hq) return;
    const int gid = lane >> 2, tig = lane & 3;
    const int g = h / p.G;

    const Unit u = resolve_unit(p, s, part, part == 0 && h == 0 && lane == 0);
    if (u.t_begin >= u.L) {
        if (part == 0 && u.L == 0) {  // empty context: zeros
            To* o = reinterpret_cast<To*>(p.out) + ((int64_t)s * p.Hq + h) * D;
            for (int i = lane; i < D; i += 32) o[i] = To(0.f);
        }
        return;
    }
    uint32_t bar0;
    uint8_t* ring = ring_setup<kWarpBytes, kDataBytes, STAGES>(smem_raw, warp, lane, bar0, &tmK, &tmV);
    const uint32_t ring_s = smem_u32(ring);

    // q as column 0 of the B operand of S^T (lanes gid = 0).
    uint32_t qb[KSTEPS][2];
    {
        const To* qr = reinterpret_cast<const To*>(p.q) + ((int64_t)s * p.Hq + h) * D + tig * (D / 4);
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
            qb[kk][0] = gid == 0 ? H::pair(qr + 4 * kk) : 0u;
            qb[kk][1] = gid == 0 ? H::pair(qr + 4 * kk + 2) : 0u;
        }
    }
    float o[NMT][4];
#pragma unroll
    for (int j = 0; j < NMT; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    float m = -INFINITY, l = 0.f;  // m warp-uniform; l a per-lane share

    const int t_begin = u.t_begin, t_end = u.t_end;
    const int ntiles = (t_end - t_begin + TT - 1) / TT;
    const int jb0 = t_begin / p.bs;
    BlockWindow win;
    win.init(p.block_tables + (int64_t)s * p.maxB, jb0, (t_end - 1) / p.bs - jb0 + 1, lane);

    auto issue = [&](int i) {
        const int t0 = t_begin + i * TT;
        int rows[HV];
        int nh = 0;  // 16-token tiles of the stage that hold tokens of the unit
#pragma unroll
        for (int hh = 0; hh < HV; ++hh) {
            const int th = t0 + hh * kTileTok;
            if (th < t_end) {  // warp-uniform
                const int blk = win.get(th / p.bs - jb0, lane, p.NB);
                rows[hh] = (blk * p.Hkv + g) * p.bs + (th % p.bs);
                nh = hh + 1;
            }
        }
        if (lane == 0) {
            const int st = i % STAGES;
            const uint32_t bar = bar0 + 8 * st;
            const uint32_t dst = ring_s + st * C::kStageBytes;
            fence_proxy_async();
            mbar_arrive_expect_tx(bar, 2 * nh * C::kTileBytes);
#pragma unroll
            for (int hh = 0; hh < HV; ++hh) {
                if (hh < nh) {
                    tma_load_2d(dst + hh * C::kTileBytes, &tmK, 0, rows[hh], bar);
                    tma_load_2d(dst + (HV + hh) * C::kTileBytes, &tmV, 0, rows[hh], bar);
                }
            }
        }
    };
    const int npre = ntiles < STAGES ? ntiles : STAGES;
    for (int i = 0; i < npre; ++i) issue(i);

    // This lane's tokens for the P V contraction (see above).
    const int vtok[4] = {2 * tig, 2 * tig + 8, 2 * tig + 1, 2 * tig + 9};

    for (int i = 0; i < ntiles; ++i) {
        const int st = i % STAGES;
        if (!ring_wait<STAGES>(bar0, i, ntiles)) return;
        const int valid = min(TT, t_end - (t_begin + i * TT));
        const uint8_t* stage = ring + st * C::kStageBytes;

        // Codes of this lane's fragments; the stage goes back to TMA once
        // both the K and the V codes are in registers.
        uint32_t kw[HV][2][KSTEPS];  // codes of rows gid and gid + 8 of each tile
        uint32_t vw[HV][4][VW];
        auto load_v = [&]() {
#pragma unroll
            for (int hh = 0; hh < HV; ++hh) {
                const int vh = valid - hh * kTileTok;  // tokens of this tile (warp-uniform)
                if (vh <= 0) continue;
                const uint8_t* vt = stage + (HV + hh) * C::kTileBytes;
                zero_tail_rows<D>(const_cast<uint8_t*>(vt), vh, lane);
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    if constexpr (VW == 4) {
                        const uint4 w = *reinterpret_cast<const uint4*>(vt + fp8_chunk<D>(vtok[t], gid));
                        vw[hh][t][0] = w.x;
                        vw[hh][t][1] = w.y;
                        vw[hh][t][2] = w.z;
                        vw[hh][t][3] = w.w;
                    } else {
                        const uint2 w = *reinterpret_cast<const uint2*>(vt + vtok[t] * D + gid * 8);
                        vw[hh][t][0] = w.x;
                        vw[hh][t][1] = w.y;
                    }
                }
            }
            __syncwarp();
            if (i + STAGES < ntiles) issue(i + STAGES);
        };
#pragma unroll
        for (int hh = 0; hh < HV; ++hh) {
            const int vh = valid - hh * kTileTok;  // tokens of this tile (warp-uniform)
            if (vh <= 0) continue;
            const uint8_t* kt = stage + hh * C::kTileBytes;
#pragma unroll
            for (int r = 0; r < 2; ++r) {
#pragma unroll
                for (int c = 0; c < KSTEPS / 4; ++c) {
                    const uint4 w = *reinterpret_cast<const uint4*>(kt + fp8_chunk<D>(r * 8 + gid, tig * (KSTEPS / 4) + c));
                    kw[hh][r][4 * c] = w.x;
                    kw[hh][r][4 * c + 1] = w.y;
                    kw[hh][r][4 * c + 2] = w.z;
                    kw[hh][r][4 * c + 3] = w.w;
                }
            }
        }
        if constexpr (!LATE_V) load_v();

        // S^T of each tile: two accumulator chains (even / odd k-steps) halve
        // the MMA dependency depth.
        float x[HV][2];  // scores of tokens gid and gid + 8 of each tile (lanes tig = 0)
        const bool live = tig == 0;
#pragma unroll
        for (int hh = 0; hh < HV; ++hh) {
            const int vh = valid - hh * kTileTok;
            x[hh][0] = x[hh][1] = -INFINITY;
            if (vh <= 0) continue;
            float sa[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
            for (int kk = 0; kk < KSTEPS; ++kk) {
                uint32_t a[4];
                e4m3x4_to_f16x2x2(kw[hh][0][kk], a[0], a[2]);
                e4m3x4_to_f16x2x2(kw[hh][1][kk], a[1], a[3]);
                mma_16816<__half>(sa[kk & 1], a, qb[kk][0], qb[kk][1]);
            }
            if (live && gid < vh) x[hh][0] = (sa[0][0] + sa[1][0]) * p.scale_log2;
            if (live && gid + 8 < vh) x[hh][1] = (sa[0][2] + sa[1][2]) * p.scale_log2;
        }
        float mt = fmaxf(x[0][0], x[0][1]);
#pragma unroll
        for (int hh = 1; hh < HV; ++hh) mt = fmaxf(mt, fmaxf(x[hh][0], x[hh][1]));
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
        const float mn = fmaxf(m, mt);
        const float b = mn == -INFINITY ? 0.f : mn;  // no -inf - -inf
        const float alpha = ex2(m - b);
        m = mn;
        if (alpha != 1.f) {  // warp-uniform; exactly 1 once the maximum settles
            l *= alpha;
#pragma unroll
            for (int j = 0; j < NMT; ++j) {
                o[j][0] *= alpha;
                o[j][2] *= alpha;
            }
        }
        if constexpr (LATE_V) load_v();
#pragma unroll
        for (int hh = 0; hh < HV; ++hh) {
            if (valid - hh * kTileTok <= 0) continue;  // warp-uniform
            const float p_lo = ex2(x[hh][0] - b), p_hi = ex2(x[hh][1] - b);
            l += p_lo + p_hi;
            // Lane (j, 0) holds the pair (token j, token j + 8) = contraction
            // indices (2j, 2j+1); lane (0, tig) gathers pairs 2tig and 2tig+1.
            const uint32_t pair = Elt<__half>::pack2(p_lo, p_hi);
            const uint32_t g0 = __shfl_sync(0xffffffffu, pair, 8 * tig);
            const uint32_t g1 = __shfl_sync(0xffffffffu, pair, 8 * tig + 4);
            const uint32_t pb0 = gid == 0 ? g0 : 0u;
            const uint32_t pb1 = gid == 0 ? g1 : 0u;

            // O^T += V^T p^T
#pragma unroll
            for (int w = 0; w < VW; ++w) {
                const uint32_t lo0 = __byte_perm(vw[hh][0][w], vw[hh][1][w], 0x5140);
                const uint32_t hi0 = __byte_perm(vw[hh][0][w], vw[hh][1][w], 0x7362);
                const uint32_t lo1 = __byte_perm(vw[hh][2][w], vw[hh][3][w], 0x5140);
                const uint32_t hi1 = __byte_perm(vw[hh][2][w], vw[hh][3][w], 0x7362);
                uint32_t a0[4], a1[4];
                e4m3x4_to_f16x2x2(lo0, a0[0], a0[1]);
                e4m3x4_to_f16x2x2(lo1, a0[2], a0[3]);
                mma_16816<__half>(o[2 * w], a0, pb0, pb1);
                e4m3x4_to_f16x2x2(hi0, a1[0], a1[1]);
                e4m3x4_to_f16x2x2(hi1, a1[2], a1[3]);
                mma_16816<__half>(o[2 * w + 1], a1, pb0, pb1);
            }
        }
    }
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) l += __shfl_xor_sync(0xffffffffu, l, off);

    // Lane (gid, 0): elements gid*SPAN + 2mt (o[mt][0]) and + 2mt + 1 (o[mt][2]).
    const int64_t row = (int64_t)s * p.Hq + h;
    if (u.direct) {
        if (tig != 0) return;
        const float inv = p.v_scale / l;
        uint32_t hw[NMT];
#pragma unroll
        for (int j = 0; j < NMT; ++j) hw[j] = Elt<To>::pack2(o[j][0] * inv, o[j][2] * inv);
        uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<To*>(p.out) + row * D + gid * SPAN);
#pragma unroll
        for (int v = 0; v < NMT / 4; ++v) dst[v] = make_uint4(hw[4 * v], hw[4 * v + 1], hw[4 * v + 2], hw[4 * v + 3]);
        return;
    }
    const unsigned long long seen = p.split_count != nullptr && lane == 0 ? split_peek(p.split_count + row) : 0ull;
    if (tig == 0) {
        const int64_t idx = row * p.maxP + u.slot;
        float4* dst = reinterpret_cast<float4*>(p.ws_o + idx * D + gid * SPAN);
#pragma unroll
        for (int v = 0; v < NMT / 2; ++v)
            dst[v] = make_float4(o[2 * v][0] * p.v_scale, o[2 * v][2] * p.v_scale, o[2 * v + 1][0] * p.v_scale,
                                 o[2 * v + 1][2] * p.v_scale);
        if (gid == 0) *reinterpret_cast<float2*>(p.ws_ml + idx * 2) = make_float2(m, l);
    }
    if (p.split_count != nullptr) merge_if_last<To, D>(p, row, u.nsuf, lane, seen);
}

}  // namespace pkv
