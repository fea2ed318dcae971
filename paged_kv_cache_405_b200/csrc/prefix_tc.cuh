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
// Per 128-token tile j of the partition and Q tile q (thread t of softmax
// warpgroup q owns query row t = TMEM lane t):
//   S = Q K^T   M = 128 rows, N = 128 tokens, K = 128 head-dim elements (8
//               MMAs of 16).  A = Q (built in shared memory from the rows'
//               query vectors, K-major, 128-byte swizzle, two 64-element
//               column blocks); B = the K tile as TMA loads it (K-major, the
//               same two blocks).
//   softmax     the thread reads its 128 scores and writes P = exp2(s - m) in
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
// One M = 128 MMA costs the tensor core about as much at N = 64 as at N =
// 128, hence tiles of 128 tokens.  The MMAs go in as units u = (j, q) in the
// order S(u0), .., S(u_{L-1}), then PV(u), S(u + L) for u = 0, 1, ..: with
// two Q tiles (L = 2, one score buffer per Q tile) the tensor core computes
// one tile's scores and the other's P V while each softmax runs; with one
// (L = 2 with two score buffers) the next tile's scores overlap the softmax.
// Rows are (sequence first + r / G, query head g*G + r % G), as in the mma.sync
// pass; rows whose sequence does not take the group's prefix result (see
// group_members_kernel) are computed from zero queries and not written.  The
// partials leave through shared memory (a row per thread at a 528-byte pitch),
// each row stored by one warp as 512 contiguous bytes.
//
// Warp roles: warps 0 .. 4*QT-1 are the softmax warpgroups (warp w reads TMEM
// lanes 32*(w % 4) ..), then one warp copies K, one V (each into its own
// two-tile ring, refilled as the MMAs release slots), and lane 0 of the last
// warp issues every MMA.  A tile's copies are two-dimensional TMA boxes (16
// tokens x 64 head-dim elements, 128-byte swizzle: two per 16-token block of
// one head), issued from 16 lanes at once.  The copies start while the
// softmax warps gather Q.  Every wait is bounded in time; a give-up records
// PKV_DEVERR_TIMEOUT and raises a CTA-wide abort flag that every other wait
// also polls; then each role waits (bounded) for what it has in flight (MMAs,
// copies), tensor memory is freed and the CTA returns.
//
// Sizes: QT = 2 (256 rows): 192 KB of shared memory, one CTA per SM; QT = 1:
// 160 KB.  Either way 512 TMEM columns and one CTA per SM, so an allocation
// never waits on another CTA of this kernel.
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

// Columns c .. c+31 (c+127) of this warp's 32 lanes (thread i of the warp:
// lane base + i); the values are complete when the call returns (the wait is
// in the same asm statement).
__device__ __forceinline__ void ld_x32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "{\n\ttcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;\n\t}"
        : PKV_TO8(0), PKV_TO8(8), PKV_TO8(16), PKV_TO8(24)
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void ld_x128(uint32_t taddr, uint32_t (&r)[128]) {
    asm volatile(
        "{\n\ttcgen05.ld.sync.aligned.32x32b.x128.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, "
        "%35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, "
        "%56, %57, %58, %59, %60, %61, %62, %63, %64, %65, %66, %67, %68, %69, %70, %71, %72, %73, %74, %75, %76, "
        "%77, %78, %79, %80, %81, %82, %83, %84, %85, %86, %87, %88, %89, %90, %91, %92, %93, %94, %95, %96, %97, "
        "%98, %99, %100, %101, %102, %103, %104, %105, %106, %107, %108, %109, %110, %111, %112, %113, %114, %115, "
        "%116, %117, %118, %119, %120, %121, %122, %123, %124, %125, %126, %127}, [%128];\n\t"
        "tcgen05.wait::ld.sync.aligned;\n\t}"
        : PKV_TO8(0), PKV_TO8(8), PKV_TO8(16), PKV_TO8(24), PKV_TO8(32), PKV_TO8(40), PKV_TO8(48), PKV_TO8(56),
          PKV_TO8(64), PKV_TO8(72), PKV_TO8(80), PKV_TO8(88), PKV_TO8(96), PKV_TO8(104), PKV_TO8(112), PKV_TO8(120)
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

// Shared memory of the pass (offsets from a 1024-byte aligned base) and
// tensor-memory columns.
template <int QT>
struct PrefixTcCfg {
    static constexpr int kTok = 128;           // tokens per K / V tile
    static constexpr int kQBlk = 128 * 128;    // 128 query rows x 64 head-dim elements (16 KB)
    static constexpr int kHalf = kTok * 128;   // 128 token rows x 64 head-dim elements (16 KB)
    static constexpr int kTile = 2 * kHalf;    // one K or V tile, both head-dim halves
    static constexpr int KS = 2, VS = 2;       // ring tiles
    static constexpr int kQOff = 0;            // Q tile q: blocks 2q, 2q+1
    static constexpr int kKOff = kQOff + QT * 2 * kQBlk;
    static constexpr int kVOff = kKOff + KS * kTile;
    static constexpr int kBarOff = kVOff + VS * kTile;
    static constexpr int kSB = QT == 1 ? 2 : 1;  // score buffers per Q tile
    static constexpr int kLook = QT * kSB;       // units whose scores go in ahead of P V
    // kfull[KS], kempty[KS], vfull[VS], vempty[VS]; per Q tile sfull[kSB],
    // pfull[kSB], obar; Q written; all MMAs done; drain
    static constexpr int kBars = 2 * KS + 2 * VS + QT * (2 * kSB + 1) + 3;
    static constexpr int kTmemOff = kBarOff + 8 * kBars;
    static constexpr int kAbortOff = kTmemOff + 4;
    static constexpr int kSmemBytes = 1024 + kAbortOff + 4;
    static constexpr int kCols = 512;
    static constexpr int kQCols = (kSB + 1) * 128;  // per Q tile: score buffers, then O
    static constexpr int kPitch = 528;               // staging row pitch of the partials (bytes)
    static constexpr int kWarps = 4 * QT + 3;        // softmax warpgroups, K copies, V copies, MMA
    static constexpr int kThreads = 32 * kWarps;
    static_assert(QT * kQCols <= kCols, "tensor-memory columns");
    static_assert(128 * QT * kPitch <= kBarOff, "staging fits below the barriers");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
    static_assert(2 * (kSmemBytes + 1024) > 228 * 1024, "one CTA per SM (tensor-memory columns)");
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

template <typename T, int QT>
__global__ void __launch_bounds__(PrefixTcCfg<QT>::kThreads, 1)
    prefix_attn_tc_kernel(const AttnParams p, const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV) {
    using C = PrefixTcCfg<QT>;
    constexpr int D = 128, TOK = C::kTok, KS = C::KS, VS = C::VS, SB = C::kSB;
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
    const uint32_t b_q = b_vempty + 8 * VS;  // Q tile q at +8(2SB+1)q: sfull[SB], pfull[SB], obar
    constexpr int kQBars = 8 * (2 * SB + 1);
    const uint32_t b_qready = b_q + kQBars * QT, b_done = b_qready + 8, b_drain = b_done + 8;
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

    // ---- set-up: tensor memory and barriers; then the copies start while
    // the softmax warps gather Q (handed to the MMA warp on b_qready)
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
            for (int b = 0; b < SB; ++b) {
                mbar_init(b_q + kQBars * i + 8 * b, 1);            // S ready
                mbar_init(b_q + kQBars * i + 8 * (SB + b), 128);   // P written: every softmax thread of the tile
            }
            mbar_init(b_q + kQBars * i + 16 * SB, 1);              // O products of a tile done
        }
        mbar_init(b_qready, 128 * QT);  // every softmax thread
        mbar_init(b_done, 1);
        mbar_init(b_drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
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
        const int nblk = (t1 - 1) / p.bs - jb0 + 1;  // table entries of the partition
        const int32_t* trow = p.block_tables + (int64_t)first * p.maxB + jb0;
        int wbase = 0;  // entries wbase .. wbase+31 of the partition: lane i holds wbase + i
        int wmine = lane < nblk ? trow[lane] : 0;
        for (int j = 0; j < n; ++j) {
            const int slot = j % S;
            if (j >= S) {
                bool w = true;
                if (lane == 0) w = mbar_wait_or_abort(empty + 8 * slot, ((j / S) - 1) & 1, abort_flag);
                if (!__shfl_sync(0xffffffffu, w ? 1 : 0, 0)) break;
            }
            const int tt0 = t0 + j * TOK;
            const int nbox = min(TOK, t1 - tt0) / kTileTok;
            const int jfirst = tt0 / p.bs - jb0, jlast = (tt0 + nbox * kTileTok - 1) / p.bs - jb0;
            if (jlast >= wbase + 32) {  // warp-uniform; a tile spans at most eight entries
                wbase = jfirst;
                wmine = wbase + lane < nblk ? trow[wbase + lane] : 0;
            }
            // lane 2b + h copies head-dim half h of box b (16 tokens; a box
            // never straddles a block, as bs % 16 == 0)
            const int b = lane >> 1, hx = lane & 1;
            const int th = tt0 + min(b, nbox - 1) * kTileTok;
            int blk = __shfl_sync(0xffffffffu, wmine, th / p.bs - jb0 - wbase);
            if ((unsigned)blk >= (unsigned)p.NB) {
                if (b < nbox) flag_error(1u /* PKV_DEVERR_BLOCK_ID */);
                blk = 0;  // read a valid block instead; the output is flagged meaningless
            }
            const uint32_t dst = ring + slot * C::kTile, bar = full + 8 * slot;
            if (lane == 0) mbar_arrive_expect_tx(bar, (uint32_t)(nbox * kTileTok * D * 2));
            __syncwarp();
            if (b < nbox)
                tma_load_2d(dst + hx * C::kHalf + b * kTileTok * 128, map, hx * 64,
                            (blk * p.Hkv + g) * p.bs + (th % p.bs), bar);
            issued = j + 1;
        }
    } else if (warp == kWarpM) {
        // ---- MMAs (lane 0) in units u = j * nq + q, once Q is in shared memory
        if (lane == 0) {
            constexpr uint32_t kIdS = tc::idesc_f16_m128<T>(128, false);
            constexpr uint32_t kIdO = tc::idesc_f16_m128<T>(128, true);
            // descriptors of the operand bases; an MMA adds its operand's
            // offset (16-byte units) to the start-address field, which stays
            // below 2^14 for shared-memory addresses
            const uint64_t qdesc0 = tc::smem_desc_sw128(sbase + C::kQOff, 16, 1024);
            const uint64_t kdesc0 = tc::smem_desc_sw128(sbase + C::kKOff, 16, 1024);
            const uint64_t vdesc0 = tc::smem_desc_sw128(sbase + C::kVOff, C::kHalf, 1024);
            const int U = n * nq, L = nq * SB;
            auto issue_s = [&](int u) -> bool {
                const int j = u / nq, qq = u - j * nq, slot = j % KS;
                if (qq == 0) {
                    if (!mbar_wait_or_abort(b_kfull + 8 * slot, (j / KS) & 1, abort_flag)) return false;
                    tc::fence_after_sync();
                }
                const uint64_t qd = qdesc0 + (uint64_t)((qq * 2 * C::kQBlk) >> 4);
                const uint64_t kd = kdesc0 + (uint64_t)((slot * C::kTile) >> 4);
                const int b = SB == 2 ? (j & 1) : 0;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    tc::mma_f16(tmem + qq * C::kQCols + b * 128,
                                qd + (uint64_t)(((kk >> 2) * C::kQBlk + (kk & 3) * 32) >> 4),
                                kd + (uint64_t)(((kk >> 2) * C::kHalf + (kk & 3) * 32) >> 4), kIdS, kk > 0);
                tc::commit(b_q + kQBars * qq + 8 * b);          // S ready
                if (qq == nq - 1) tc::commit(b_kempty + 8 * slot);  // K slot free
                return true;
            };
            auto issue_pv = [&](int u) -> bool {
                const int j = u / nq, qq = u - j * nq, slot = j % VS;
                if (qq == 0) {
                    if (!mbar_wait_or_abort(b_vfull + 8 * slot, (j / VS) & 1, abort_flag)) return false;
                }
                const int b = SB == 2 ? (j & 1) : 0;
                if (!mbar_wait_or_abort(b_q + kQBars * qq + 8 * (SB + b), (j / SB) & 1, abort_flag)) return false;
                tc::fence_after_sync();
                const int valid = min(TOK, t1 - (t0 + j * TOK));
                const uint64_t vd = vdesc0 + (uint64_t)((slot * C::kTile) >> 4);
                for (int kk = 0; kk < valid / 16; ++kk)
                    tc::mma_f16_tmem_a(tmem + qq * C::kQCols + SB * 128, tmem + qq * C::kQCols + b * 128 + kk * 8,
                                       vd + (uint64_t)((kk * 16 * 128) >> 4), kIdO, j > 0 || kk > 0);
                tc::commit(b_q + kQBars * qq + 16 * SB);             // O products of tile j done
                if (qq == nq - 1) tc::commit(b_vempty + 8 * slot);  // V slot free
                return true;
            };
            bool ok = mbar_wait_or_abort(b_qready, 0, abort_flag);
            for (int u = 0; ok && u < min(L, U); ++u) ok = issue_s(u);
            for (int u = 0; ok && u < U; ++u) {
                ok = issue_pv(u);
                if (ok && u + L < U) ok = issue_s(u + L);
            }
            if (ok) tc::commit(b_done);  // every product done
            // every MMA issued, and so every arrival it owes, has completed
            // before the CTA can leave (bounded)
            tc::commit(b_drain);
            mbar_wait(b_drain, 0);
        }
        __syncwarp();
    } else {
        // ---- softmax warps: gather Q, then tile q's softmax (thread t owns row t)
        const bool live = inrow && p.member[s_r].x == gi + 1;
        if (q < nq) {
            const uint4* qsrc = reinterpret_cast<const uint4*>(reinterpret_cast<const T*>(p.q) +
                                                                 ((int64_t)s_r * p.Hq + h_r) * D);
            uint8_t* qrow = smem + C::kQOff + q * 2 * C::kQBlk + t * 128;
            uint4 v[16];  // all loads in flight before the first store
#pragma unroll
            for (int c = 0; c < 16; ++c) v[c] = live ? __ldg(qsrc + c) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int c = 0; c < 16; ++c)  // 16-byte chunk c: block c / 8, chunk c % 8 of the row
                *reinterpret_cast<uint4*>(qrow + (c >> 3) * C::kQBlk + (((c & 7) ^ (t & 7)) << 4)) = v[c];
            fence_proxy_async();  // the generic Q writes, before the tensor core reads them
        }
        mbar_arrive(b_qready);
        if (q < nq) {
            const uint32_t tq = tmem + ((uint32_t)((warp & 3) * 32) << 16) + q * C::kQCols;
            const uint32_t sfull = b_q + kQBars * q, pfull = sfull + 8 * SB, obar = sfull + 16 * SB;
            const float sl2 = p.scale_log2;  // >= 0
            float m = -INFINITY, l = 0.f;
            bool ok = true;
            for (int j = 0; j < n; ++j) {
                const int b = SB == 2 ? (j & 1) : 0;
                const uint32_t sc = tq + b * 128;
                const bool w = mbar_wait_or_abort(sfull + 8 * b, (j / SB) & 1, abort_flag);
                if (!__all_sync(0xffffffffu, w)) {
                    ok = false;
                    break;
                }
                tc::fence_after_sync();
                const int valid = min(TOK, t1 - (t0 + j * TOK));  // a multiple of 16
                uint32_t a[128];
                tc::ld_x128(sc, a);
                float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                for (int k = 0; k < 128; k += 4)
                    if (k < valid) {
#pragma unroll
                        for (int i = 0; i < 4; ++i) mx[i] = fmaxf(mx[i], __uint_as_float(a[k + i]));
                    }
                const float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * sl2;
                const bool need = mt > m + kPrefixRescaleLog2;  // always on the first tile
                const float mn = need ? mt : m;
                const float alpha = ex2(m - mn);  // 1 when m stays; 0 on the first tile (m = -inf)
                if (j > 0 && __any_sync(0xffffffffu, need)) {
                    // the previous tile's O products must have landed before O is rescaled
                    const bool w2 = mbar_wait_or_abort(obar, (j - 1) & 1, abort_flag);
                    if (!__all_sync(0xffffffffu, w2)) {
                        ok = false;
                        break;
                    }
                    tc::fence_after_sync();
#pragma unroll 1
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t o[32];
                        tc::ld_x32(tq + SB * 128 + c * 32, o);
#pragma unroll
                        for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
                        tc::st_x32(tq + SB * 128 + c * 32, o);
                    }
                }
                float lsum[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int h = 0; h < 2; ++h) {  // P of tokens k, k+1 into score column k / 2
                    uint32_t pw[32];
#pragma unroll
                    for (int k = 64 * h; k < 64 * h + 64; k += 2) {
                        const float p0 = k < valid ? ex2(fmaf(__uint_as_float(a[k]), sl2, -mn)) : 0.f;
                        const float p1 = k < valid ? ex2(fmaf(__uint_as_float(a[k + 1]), sl2, -mn)) : 0.f;
                        lsum[(k >> 1) & 3] += p0 + p1;
                        pw[(k >> 1) & 31] = Elt<T>::pack2(p0, p1);
                    }
                    tc::st_x32(sc + 32 * h, pw);
                }
                const float ls = (lsum[0] + lsum[1]) + (lsum[2] + lsum[3]);
                l = l * alpha + ls;
                m = mn;
                tc::fence_before_sync();
                mbar_arrive(pfull + 8 * b);
            }
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait_or_abort(b_done, 0, abort_flag));
            if (ok) {
                // ---- the row's partial: o (unnormalised, at reference maximum m), m, l;
                // every MMA is done, so Q and the rings are free for staging
                tc::fence_after_sync();
                uint8_t* stage = smem + (q * 128 + t) * C::kPitch;
#pragma unroll 1
                for (int cc = 0; cc < D / 32; ++cc) {
                    uint32_t o[32];
                    tc::ld_x32(tq + SB * 128 + cc * 32, o);
#pragma unroll
                    for (int k = 0; k < 32; k += 4)
                        *reinterpret_cast<uint4*>(stage + (cc * 32 + k) * 4) = make_uint4(o[k], o[k + 1], o[k + 2], o[k + 3]);
                }
                const int64_t idx = ((int64_t)s_r * p.Hq + h_r) * p.maxP + pp;
                if (live) *reinterpret_cast<float2*>(p.ws_ml + idx * 2) = make_float2(m, l);
                __syncwarp();  // this warp's 32 rows are staged
                // one row per step, 512 contiguous bytes: lane i stores bytes 16i .. 16i+15
                const uint8_t* wstage = smem + (q * 128 + (warp & 3) * 32) * C::kPitch;
#pragma unroll 4
                for (int i = 0; i < 32; ++i) {
                    const int64_t idx_i = __shfl_sync(0xffffffffu, idx, i);
                    if (__shfl_sync(0xffffffffu, live ? 1 : 0, i))
                        *reinterpret_cast<uint4*>(p.ws_o + idx_i * D + lane * 4) =
                            *reinterpret_cast<const uint4*>(wstage + i * C::kPitch + lane * 16);
                }
            }
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
