// Paged decode attention for grouped-query attention on tensor cores: one
// warp per (sequence, kv head, partition) serves all G query heads of the
// group (2 <= G <= 16), so each K/V byte is read once for G queries and the
// work is a real (G x D) . (D x tokens) contraction.
//
// Per 16-token tile (tokens of one block, via the block table; openeuler.csdn.net
// PagedAttention explainer 4.2, aiknowledge.cn "2.2 PagedAttention 与 KV
// Cache 分页管理" 2.2.3-2.2.4):
//   S = Q K^T   : m16n8k16 MMAs, A = Q (the G heads padded to 16 rows, held in
//                 registers for the whole unit), B = K^T straight from the
//                 shared-memory tile (ldmatrix; a K row is a "column" of B).
//   online softmax on the accumulator fragments (rows = heads; each row is
//                 spread over the 4 lanes of a quad), log2 domain.
//   O += P V    : P re-packed from the S accumulators into A fragments without
//                 touching memory; B = V via ldmatrix.trans.
//
// Data movement: each stage is one 16-token tile of K and one of V, brought in
// by 2-D tensor TMA (box 64 elements x 16 rows) with 128-byte swizzle, so the
// 8 rows an ldmatrix reads fall in 8 different bank groups.  The tensor maps
// view a pool as a matrix of (num_blocks*Hkv*block_size) rows of D elements;
// row (block*Hkv + g)*block_size + offset is the token's K (or V) row.
#pragma once
#include "attention_common.cuh"

namespace pkv {

template <typename T, int D, int WARPS, int STAGES>
struct MmaCfg {
    static constexpr int kHalfTile = kTileTok * 128;        // 16 rows x 64 elements (bytes)
    static constexpr int kTileBytes = kTileTok * D * 2;     // one K (or V) tile
    static constexpr int kStageBytes = 2 * kTileBytes;
    static constexpr int kDataBytes = WARPS * STAGES * kStageBytes;
    static constexpr int kSmemBytes = 1024 + kDataBytes + WARPS * STAGES * 8;  // + alignment slack
    static_assert(D % 64 == 0, "head_dim must be a multiple of 64");
};

template <typename T, int D, int WARPS, int STAGES>
__global__ void __launch_bounds__(WARPS * 32) paged_attn_mma_kernel(const AttnParams p,
                                                                    const __grid_constant__ CUtensorMap tmK,
                                                                    const __grid_constant__ CUtensorMap tmV) {
    using C = MmaCfg<T, D, WARPS, STAGES>;
    constexpr int KSTEPS = D / 16;  // MMA k-steps over head_dim
    constexpr int NT_O = D / 8;     // output n-tiles
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g = blockIdx.x * WARPS + warp;  // kv head
    const int part = blockIdx.y;
    const int s = blockIdx.z;
    if (g >= p.Hkv) return;

    const int gid = lane >> 2;  // accumulator row (query head within the group) and row+8
    const int tig = lane & 3;
    const int G = p.G;
    const int h0 = g * G;

    const int L = load_context_len(p, s, part == 0 && g == 0 && lane == 0);
    const int nP = (L + p.P - 1) / p.P;
    const int t_begin = part * p.P;
    if (t_begin >= L) {
        if (part == 0) {  // empty context: zeros for the group's heads
            T* o = reinterpret_cast<T*>(p.out) + ((int64_t)s * p.Hq + h0) * D;
            for (int i = lane; i < G * D; i += 32) o[i] = T(0.f);
        }
        return;
    }
    const int t_end = min(L, t_begin + p.P);
    const int ntiles = (t_end - t_begin + kTileTok - 1) / kTileTok;

    uint8_t* ring = smem + warp * STAGES * C::kStageBytes;
    const uint32_t ring_s = smem_u32(ring);
    const uint32_t bar0 = smem_u32(smem + C::kDataBytes + warp * STAGES * 8);
    if (lane == 0) {
        prefetch_tensor_map(&tmK);
        prefetch_tensor_map(&tmV);
        for (int i = 0; i < STAGES; ++i) mbar_init(bar0 + 8 * i, 1);
        fence_barrier_init();
    }
    __syncwarp();

    // Q fragments (A operand, rows = heads of the group, zero past G).
    uint32_t qa[KSTEPS][4];
    {
        const T* qb = reinterpret_cast<const T*>(p.q) + ((int64_t)s * p.Hq + h0) * D;
        const bool r0 = gid < G, r1 = gid + 8 < G;
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
            const int c0 = kk * 16 + 2 * tig;
            qa[kk][0] = r0 ? *reinterpret_cast<const uint32_t*>(qb + gid * D + c0) : 0u;
            qa[kk][1] = r1 ? *reinterpret_cast<const uint32_t*>(qb + (gid + 8) * D + c0) : 0u;
            qa[kk][2] = r0 ? *reinterpret_cast<const uint32_t*>(qb + gid * D + c0 + 8) : 0u;
            qa[kk][3] = r1 ? *reinterpret_cast<const uint32_t*>(qb + (gid + 8) * D + c0 + 8) : 0u;
        }
    }

    const int jb0 = t_begin / p.bs;
    BlockWindow win;
    win.init(p.block_tables + (int64_t)s * p.maxB, jb0, (t_end - 1) / p.bs - jb0 + 1, lane);

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
                tma_load_2d(dst + hx * C::kHalfTile, &tmK, hx * 64, row, bar);
                tma_load_2d(dst + C::kTileBytes + hx * C::kHalfTile, &tmV, hx * 64, row, bar);
            }
        }
    };

    const int npre = ntiles < STAGES ? ntiles : STAGES;
    for (int i = 0; i < npre; ++i) issue(i);

    // Per-lane ldmatrix row addresses (byte offsets inside a tile).
    const int mi = lane >> 3, ri = lane & 7;
    const int k_tok = (mi >> 1) * 8 + ri;  // K: matrices (tok 0-7|8-15) x (d lo|hi)
    const int k_hi = mi & 1;
    const int v_tok = (mi & 1) * 8 + ri;   // V (trans): (tok lo|hi) x (d lo|hi)
    const int v_hi = mi >> 1;

    float oacc[NT_O][4];
#pragma unroll
    for (int j = 0; j < NT_O; ++j) oacc[j][0] = oacc[j][1] = oacc[j][2] = oacc[j][3] = 0.f;
    float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.f, l_hi = 0.f;

    for (int i = 0; i < ntiles; ++i) {
        const int st = i % STAGES;
        const bool ok = mbar_wait(bar0 + 8 * st, (i / STAGES) & 1);
        if (!__all_sync(0xffffffffu, ok)) {
            for (int k = i + 1; k < ntiles && k < i + STAGES; ++k) mbar_wait(bar0 + 8 * (k % STAGES), (k / STAGES) & 1);
            return;
        }
        const int valid = min(kTileTok, t_end - (t_begin + i * kTileTok));
        const uint32_t Ks = ring_s + st * C::kStageBytes;
        const uint32_t Vs = Ks + C::kTileBytes;

        // S = Q K^T  (16 heads x 16 tokens as two n-tiles of 8 tokens)
        float sacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
            const int chunk = kk * 2 + k_hi;
            const uint32_t addr = Ks + (chunk >> 3) * C::kHalfTile + k_tok * 128 + (((chunk & 7) ^ (k_tok & 7)) << 4);
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4(addr, b0, b1, b2, b3);
            mma_16816<T>(sacc[0], qa[kk], b0, b1);
            mma_16816<T>(sacc[1], qa[kk], b2, b3);
        }

        // Online softmax.  Element e of n-tile nt is token nt*8 + 2*tig + (e&1),
        // head row gid (e<2) or gid+8 (e>=2).
        float mx_lo = -INFINITY, mx_hi = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int tok = nt * 8 + 2 * tig + (e & 1);
                const float x = tok < valid ? sacc[nt][e] * p.scale_log2 : -INFINITY;
                sacc[nt][e] = x;
                if (e < 2) mx_lo = fmaxf(mx_lo, x);
                else mx_hi = fmaxf(mx_hi, x);
            }
        }
#pragma unroll
        for (int off = 1; off < 4; off <<= 1) {
            mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, off));
            mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, off));
        }
        const float mn_lo = fmaxf(m_lo, mx_lo), mn_hi = fmaxf(m_hi, mx_hi);
        const float a_lo = ex2(m_lo - mn_lo), a_hi = ex2(m_hi - mn_hi);
        m_lo = mn_lo;
        m_hi = mn_hi;
        float ps_lo = 0.f, ps_hi = 0.f;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float pr = ex2(sacc[nt][e] - (e < 2 ? mn_lo : mn_hi));
                sacc[nt][e] = pr;
                if (e < 2) ps_lo += pr;
                else ps_hi += pr;
            }
        }
        l_lo = l_lo * a_lo + ps_lo;
        l_hi = l_hi * a_hi + ps_hi;
#pragma unroll
        for (int j = 0; j < NT_O; ++j) {
            oacc[j][0] *= a_lo;
            oacc[j][1] *= a_lo;
            oacc[j][2] *= a_hi;
            oacc[j][3] *= a_hi;
        }
        uint32_t pa[4];
        pa[0] = Elt<T>::pack2(sacc[0][0], sacc[0][1]);
        pa[1] = Elt<T>::pack2(sacc[0][2], sacc[0][3]);
        pa[2] = Elt<T>::pack2(sacc[1][0], sacc[1][1]);
        pa[3] = Elt<T>::pack2(sacc[1][2], sacc[1][3]);

        // Rows past the context may hold anything (even NaN): zero them in V so
        // that 0-weights cannot turn into NaN inside the MMA.
        if (valid < kTileTok) {
            uint8_t* vrow = ring + st * C::kStageBytes + C::kTileBytes;
            for (int idx = lane; idx < (kTileTok - valid) * (D / 8); idx += 32) {
                const int r = valid + idx / (D / 8);
                const int q16 = idx % (D / 8);  // 16-byte unit in the row (any order)
                *reinterpret_cast<uint4*>(vrow + (q16 >> 3) * C::kHalfTile + r * 128 + (q16 & 7) * 16) =
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
            mma_16816<T>(oacc[2 * jj], pa, b0, b1);
            mma_16816<T>(oacc[2 * jj + 1], pa, b2, b3);
        }
        __syncwarp();
        if (i + STAGES < ntiles) issue(i + STAGES);
    }

#pragma unroll
    for (int off = 1; off < 4; off <<= 1) {
        l_lo += __shfl_xor_sync(0xffffffffu, l_lo, off);
        l_hi += __shfl_xor_sync(0xffffffffu, l_hi, off);
    }
    const bool w_lo = gid < G, w_hi = gid + 8 < G;
    if (nP == 1) {
        const float i_lo = 1.f / l_lo, i_hi = 1.f / l_hi;
        T* ob = reinterpret_cast<T*>(p.out) + ((int64_t)s * p.Hq + h0) * D;
#pragma unroll
        for (int j = 0; j < NT_O; ++j) {
            const int d = j * 8 + 2 * tig;
            if (w_lo) *reinterpret_cast<uint32_t*>(ob + gid * D + d) = Elt<T>::pack2(oacc[j][0] * i_lo, oacc[j][1] * i_lo);
            if (w_hi)
                *reinterpret_cast<uint32_t*>(ob + (gid + 8) * D + d) = Elt<T>::pack2(oacc[j][2] * i_hi, oacc[j][3] * i_hi);
        }
    } else {
        const int64_t i_lo = ((int64_t)s * p.Hq + h0 + gid) * p.maxP + part;
        const int64_t i_hi = ((int64_t)s * p.Hq + h0 + gid + 8) * p.maxP + part;
#pragma unroll
        for (int j = 0; j < NT_O; ++j) {
            const int d = j * 8 + 2 * tig;
            if (w_lo) *reinterpret_cast<float2*>(p.ws_o + i_lo * D + d) = make_float2(oacc[j][0], oacc[j][1]);
            if (w_hi) *reinterpret_cast<float2*>(p.ws_o + i_hi * D + d) = make_float2(oacc[j][2], oacc[j][3]);
        }
        if (tig == 0) {
            if (w_lo) *reinterpret_cast<float2*>(p.ws_ml + i_lo * 2) = make_float2(m_lo, l_lo);
            if (w_hi) *reinterpret_cast<float2*>(p.ws_ml + i_hi * 2) = make_float2(m_hi, l_hi);
        }
    }
}

}  // namespace pkv
