// pagedkv C ABI: argument checking, launch configuration and dispatch for the
// device calls declared in include/pagedkv.h.  One translation unit holds all
// kernels so that they share the device error word.
#include <algorithm>
#include <atomic>
#include <climits>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <random>
#include <chrono>
#include <string>
#include <utility>

#include <cudaTypedefs.h>

#include "../../include/pagedkv.h"
#include "attention_fp8.cuh"
#include "attention_fp8_tc.cuh"
#include "prefix_tc.cuh"
#include "attention_mma.cuh"
#include "attention_simt.cuh"
#include "block_copy.cuh"
#include "kv_append.cuh"
#include "reduce.cuh"

namespace pkv_host {

thread_local std::string g_msg;
std::atomic<uint64_t> g_launches{0};

void set_error(const std::string& msg) { g_msg = msg; }

static pkv_status invalid(const char* msg) {
    g_msg = msg;
    return PKV_ERR_INVALID;
}

static pkv_status cuda_fail(const char* where, cudaError_t e) {
    g_msg = std::string(where) + ": " + cudaGetErrorString(e);
    return PKV_ERR_CUDA;
}

static bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

static int elem_size(pkv_dtype dt) { return dt == PKV_F32 ? 4 : dt == PKV_FP8_E4M3 ? 1 : 2; }

static bool valid_dtype(int dt) { return dt == PKV_F32 || dt == PKV_BF16 || dt == PKV_F16; }

static bool valid_block_size(int bs) { return bs == 16 || bs == 32 || bs == 64 || bs == 128 || bs == 256; }

static int num_sms() {
    static int n = 0;
    if (n == 0) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            n = 148;
    }
    return n;
}

// Partition size in tokens.  Explicit sizes are used as given.  The library's
// own choice splits a context only when it is long: units of at most 512
// tokens keep per-warp work short enough for the CTA scheduler to balance
// ragged lengths, and never go below kMinAutoPartition.
constexpr int kMinAutoPartition = 256;

static int choose_partition(int max_len, int requested) {
    if (requested > 0) return requested;
    const int whole = std::max(16, (max_len + 15) / 16 * 16);
    if (max_len <= 512) return whole;
    return 512;
}

// Bytes of split-K partials for rows x slots x (D + 2) floats; SIZE_MAX when
// the product does not fit in size_t (no buffer is that large, so every
// size check against it fails).
static size_t partials_bytes(int64_t rows, int64_t slots, int D) {
    size_t a = 0, b = 0, c = 0;
    if (rows < 0 || slots < 0 || D < 0) return SIZE_MAX;
    if (__builtin_mul_overflow((size_t)rows, (size_t)slots, &a) ||
        __builtin_mul_overflow(a, (size_t)D + 2, &b) || __builtin_mul_overflow(b, sizeof(float), &c))
        return SIZE_MAX;
    return c;
}

// Split-K workspace of a call without shared-prefix groups: the partials
// (rows x partitions x D floats of o, then 2 floats of (m, l) each), then,
// from the next 256-byte boundary, one 8-byte split counter per row
// (pkv::split_arrive) for kernels that merge their own partials.
static size_t split_counters_offset(size_t partials) { return (partials + 255) / 256 * 256; }

static size_t workspace_for(int S, int Hq, int D, int max_len, int P) {
    const int64_t maxP = ((int64_t)max_len + P - 1) / P;
    if (maxP <= 1) return 0;
    const size_t parts = partials_bytes((int64_t)S * Hq, maxP, D);
    const size_t counters = (size_t)S * (size_t)Hq * sizeof(unsigned long long);
    if (parts > SIZE_MAX - 256 || split_counters_offset(parts) > SIZE_MAX - counters) return SIZE_MAX;
    return split_counters_offset(parts) + counters;
}

// A 48-bit stamp per decode call (pkv::split_arrive), starting from a random
// value in each process.
static unsigned long long next_call_stamp() {
    static std::atomic<unsigned long long> next{[] {
        std::random_device rd;
        return ((unsigned long long)rd() << 32) ^ (unsigned long long)rd() ^
               (unsigned long long)std::chrono::steady_clock::now().time_since_epoch().count();
    }()};
    return next.fetch_add(1) & ((1ull << 48) - 1);
}

// Shared-prefix mode: one more partial slot per (sequence, head) than
// partitions, since a member's prefix and suffix partitions can each end
// part-way through a partition; then the per-sequence membership (8 bytes
// per sequence, see group_members_kernel).
static size_t shared_workspace_for(int S, int Hq, int D, int max_len, int P) {
    const int64_t slots = ((int64_t)max_len + P - 1) / P + 1;
    const size_t parts = partials_bytes((int64_t)S * Hq, slots, D);
    const size_t members = ((size_t)S * sizeof(int2) + 255) / 256 * 256;
    return parts > SIZE_MAX - members ? SIZE_MAX : parts + members;
}

// Smallest partition the library's own choice can produce for max_len: the
// workspace queries size for it, so the buffer fits whatever is chosen.
static int partition_bound(int max_len, int requested) {
    const int P = choose_partition(max_len, requested);
    if (requested == 0 && P < max_len) return std::min(P, kMinAutoPartition);
    return P;
}

// --------------------------------------------------------------- tensor maps
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q;
        void* f = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

// A pool as a (rows x D) matrix.  swizzled: box = 128 bytes of a row (64
// 16-bit elements or 128 FP8 codes) x 16 rows, 128-byte swizzle (tensor-core
// kernels).  Otherwise: box = D elements x tile rows, no swizzle (a plain
// row-major copy of the tile).
static bool make_pool_map(CUtensorMap* map, const void* pool, int64_t rows, int D, pkv_dtype dt, bool swizzled,
                          int tile_rows = pkv::kTileTok) {
    auto fn = encode_fn();
    if (!fn) return false;
    const int esz = elem_size(dt);
    cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)D * esz};
    cuuint32_t box[2] = {swizzled ? (cuuint32_t)(128 / esz) : (cuuint32_t)D,
                         (cuuint32_t)(swizzled ? pkv::kTileTok : tile_rows)};
    cuuint32_t estr[2] = {1, 1};
    const CUtensorMapDataType ty = dt == PKV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                   : dt == PKV_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                   : dt == PKV_FP8_E4M3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                                        : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    CUresult r = fn(map, ty, 2, const_cast<void*>(pool), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzled ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------ launch helpers
template <typename Kern>
static cudaError_t set_smem(Kern k, int bytes) {
    return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

// Launch a kernel and count it (pkv_launch_count).  Plain stream order: a
// kernel starts after the previous one on its stream has finished.  (Letting
// it be scheduled early -- programmatic dependent launch -- measured 1-2 %
// slower on the long calls here and no faster on the short ones.)
template <typename... KArgs, typename... Args>
static cudaError_t launch_k(void (*k)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                            Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = nullptr;
    cfg.numAttrs = 0;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, k, std::forward<Args>(args)...);
    if (e == cudaSuccess) g_launches++;
    return e;
}

// Launch shapes (warps per CTA, pipeline stages per warp); build-time tunables.
#ifndef PKV_SIMT_WARPS
#define PKV_SIMT_WARPS 4
#endif
#ifndef PKV_SIMT_STAGES
#define PKV_SIMT_STAGES 2
#endif
#ifndef PKV_SIMT_TILE
#define PKV_SIMT_TILE 16
#endif
#ifndef PKV_SIMT_TENSOR
#define PKV_SIMT_TENSOR 0
#endif
#ifndef PKV_MMA_WARPS
#define PKV_MMA_WARPS 4
#endif
#ifndef PKV_MMA_STAGES
#define PKV_MMA_STAGES 2
#endif
constexpr int kSimtWarps = PKV_SIMT_WARPS, kSimtStages = PKV_SIMT_STAGES, kSimtTile = PKV_SIMT_TILE;
constexpr int kMmaWarps = PKV_MMA_WARPS, kMmaStages = PKV_MMA_STAGES;
// Ring depth of the shared-prefix pass.
#ifndef PKV_PREFIX_STAGES
#define PKV_PREFIX_STAGES 2
#endif
constexpr int kPrefixStages = PKV_PREFIX_STAGES;

template <typename T, int D>
static cudaError_t launch_simt(const pkv::AttnParams& p, dim3 grid, cudaStream_t st) {
    using C = pkv::SimtCfg<T, D, kSimtWarps, kSimtStages, kSimtTile>;
    constexpr bool kTensor = PKV_SIMT_TENSOR != 0;
    auto k = pkv::paged_attn_simt_kernel<T, D, kSimtWarps, kSimtStages, kSimtTile, kTensor>;
    static cudaError_t attr = set_smem(k, C::kSmemBytes);
    if (attr != cudaSuccess) return attr;
    CUtensorMap mk, mv;
    if (kTensor) {
        const pkv_dtype dt = std::is_same<T, float>::value ? PKV_F32
                             : std::is_same<T, __half>::value ? PKV_F16 : PKV_BF16;
        const int64_t rows = (int64_t)p.NB * p.Hkv * p.bs;
        if (!make_pool_map(&mk, p.k_pool, rows, D, dt, false, kSimtTile) ||
            !make_pool_map(&mv, p.v_pool, rows, D, dt, false, kSimtTile))
            return cudaErrorInvalidValue;
    } else {
        std::memset(&mk, 0, sizeof mk);
        std::memset(&mv, 0, sizeof mv);
    }
    return launch_k(k, grid, dim3(kSimtWarps * 32), C::kSmemBytes, st, p, mk, mv);
}

template <typename T, int D>
static cudaError_t launch_mma(const pkv::AttnParams& p, dim3 grid, const CUtensorMap& mk, const CUtensorMap& mv,
                              cudaStream_t st) {
    using C = pkv::MmaCfg<T, D, kMmaWarps, kMmaStages>;
    auto k = pkv::paged_attn_mma_kernel<T, D, kMmaWarps, kMmaStages>;
    static cudaError_t attr = set_smem(k, C::kSmemBytes);
    if (attr != cudaSuccess) return attr;
    return launch_k(k, grid, dim3(kMmaWarps * 32), C::kSmemBytes, st, p, mk, mv);
}

// Shared-prefix pass at head_dim 128: on tcgen05 (default), or with
// PKV_PREFIX_TC=0 the mma.sync pass that head_dim 64 always uses.
#ifndef PKV_PREFIX_TC
#define PKV_PREFIX_TC 1
#endif

template <typename T, int QT>
static cudaError_t launch_prefix_tc_q(const pkv::AttnParams& p, int npre, const CUtensorMap& mk, const CUtensorMap& mv,
                                      cudaStream_t st) {
    using C = pkv::PrefixTcCfg<QT>;
    auto k = pkv::prefix_attn_tc_kernel<T, QT>;
    static cudaError_t attr = set_smem(k, C::kSmemBytes);
    if (attr != cudaSuccess) return attr;
    const int rows = p.max_group_size * p.G;
    const dim3 grid((rows + 128 * QT - 1) / (128 * QT), npre, p.num_groups * p.Hkv);
    return launch_k(k, grid, dim3(C::kThreads), C::kSmemBytes, st, p, mk, mv);
}

// Groups of more than 128 rows: two Q tiles per CTA share every K/V tile.
template <typename T>
static cudaError_t launch_prefix_tc(const pkv::AttnParams& p, int npre, const CUtensorMap& mk, const CUtensorMap& mv,
                                    cudaStream_t st) {
    return p.max_group_size * p.G > 128 ? launch_prefix_tc_q<T, 2>(p, npre, mk, mv, st)
                                        : launch_prefix_tc_q<T, 1>(p, npre, mk, mv, st);
}

template <typename T, int D>
static cudaError_t launch_prefix(const pkv::AttnParams& p, dim3 grid, const CUtensorMap& mk, const CUtensorMap& mv,
                                 cudaStream_t st) {
    using C = pkv::MmaCfg<T, D, kMmaWarps, kPrefixStages>;
    auto k = pkv::prefix_attn_mma_kernel<T, D, kMmaWarps, kPrefixStages>;
    static cudaError_t attr = set_smem(k, C::kSmemBytes);
    if (attr != cudaSuccess) return attr;
    return launch_k(k, grid, dim3(kMmaWarps * 32), C::kSmemBytes, st, p, mk, mv);
}

// Many partitions: 8 warps on each (sequence, head); few: 8 rows per CTA,
// one warp each.
template <typename T, int D>
static cudaError_t launch_chunk(const pkv::AttnParams& p, const pkv::ChunkParams& c, dim3 grid,
                                const CUtensorMap& mk, const CUtensorMap& mv, cudaStream_t st) {
    using C = pkv::MmaCfg<T, D, kMmaWarps, kMmaStages>;
    auto k = pkv::chunk_attn_mma_kernel<T, D, kMmaWarps, kMmaStages>;
    static cudaError_t attr = set_smem(k, C::kSmemBytes);
    if (attr != cudaSuccess) return attr;
    return launch_k(k, grid, dim3(kMmaWarps * 32), C::kSmemBytes, st, p, c, mk, mv);
}

// FP8 pools: stages of E4M3 tiles per warp, widened to FP16 in registers.
#ifndef PKV_FP8_STAGES
#define PKV_FP8_STAGES 2
#endif
constexpr int kFp8Stages = PKV_FP8_STAGES;


template <typename To, int D, bool HI>
static cudaError_t launch_mma_fp8_rows(const pkv::AttnParams& p, dim3 grid, const CUtensorMap& mk,
                                       const CUtensorMap& mv, cudaStream_t st) {
    using C = pkv::Fp8Cfg<D, kMmaWarps, kFp8Stages>;
    auto k = pkv::paged_attn_fp8_kernel<D, kMmaWarps, kFp8Stages, To, HI>;
    static cudaError_t attr = set_smem(k, C::kSmemBytes);
    if (attr != cudaSuccess) return attr;
    return launch_k(k, grid, dim3(kMmaWarps * 32), C::kSmemBytes, st, p, mk, mv);
}

// Groups of at most 8 heads leave MMA rows 8..15 empty: a variant skips them.
template <typename To, int D>
static cudaError_t launch_mma_fp8(const pkv::AttnParams& p, dim3 grid, const CUtensorMap& mk, const CUtensorMap& mv,
                                  cudaStream_t st) {
    return p.G > 8 ? launch_mma_fp8_rows<To, D, true>(p, grid, mk, mv, st)
                   : launch_mma_fp8_rows<To, D, false>(p, grid, mk, mv, st);
}

// Per-head FP8 kernel: tokens per pipeline stage (16 or 32) and CTAs per SM
// it is compiled for; build-time tunables.
#ifndef PKV_FP8_HEAD_TT
#define PKV_FP8_HEAD_TT 16
#endif
#ifndef PKV_FP8_HEAD_MINB
#define PKV_FP8_HEAD_MINB 4
#endif
#ifndef PKV_FP8_HEAD_LATE_V
#define PKV_FP8_HEAD_LATE_V 0
#endif

template <typename To, int D>
static cudaError_t launch_head_fp8(const pkv::AttnParams& p, dim3 grid, const CUtensorMap& mk, const CUtensorMap& mv,
                                   cudaStream_t st) {
    constexpr int TT = PKV_FP8_HEAD_TT;
    using C = pkv::Fp8HeadCfg<D, TT>;
    constexpr int kSmem = 1024 + kMmaWarps * kFp8Stages * (C::kStageBytes + 8);
    auto k = pkv::paged_attn_fp8_head_kernel<D, kMmaWarps, kFp8Stages, To, TT, PKV_FP8_HEAD_MINB,
                                             PKV_FP8_HEAD_LATE_V != 0>;
    static cudaError_t attr = set_smem(k, kSmem);
    if (attr != cudaSuccess) return attr;
    return launch_k(k, grid, dim3(kMmaWarps * 32), kSmem, st, p, mk, mv);
}

// Side stream for the shared-prefix pass, which runs concurrently with the
// same call's decode kernel: both only read the pools and write disjoint
// partial slots, and the reduce waits for both.  One stream and a fork / join
// event pair per device, created on first use (no device memory); the mutex
// keeps one call's fork ... join sequence from interleaving with another
// thread's.  Without them the pass runs on the caller's stream first.
struct SideStream {
    cudaStream_t stream = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
    bool tried = false, ok = false;
};
constexpr int kMaxSideDevices = 64;
static SideStream g_side[kMaxSideDevices];
static std::mutex g_side_mu;

static SideStream* side_stream() {  // the caller holds g_side_mu
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxSideDevices) {
        cudaGetLastError();
        return nullptr;
    }
    SideStream& s = g_side[dev];
    if (!s.tried) {
        s.tried = true;
        s.ok = cudaStreamCreateWithFlags(&s.stream, cudaStreamNonBlocking) == cudaSuccess &&
               cudaEventCreateWithFlags(&s.fork, cudaEventDisableTiming) == cudaSuccess &&
               cudaEventCreateWithFlags(&s.join, cudaEventDisableTiming) == cudaSuccess;
        if (!s.ok) cudaGetLastError();  // fall back to the caller's stream
    }
    return s.ok ? &s : nullptr;
}

template <typename T, int D>
static cudaError_t launch_reduce(const pkv::ReduceParams& r, cudaStream_t st) {
    const unsigned rows = (unsigned)((r.query_start ? r.T : r.S) * r.Hq);
    if (r.maxP > 32) return launch_k(pkv::splitk_reduce_kernel<T, D, 8, 1>, dim3(rows), dim3(256), 0, st, r);
    const dim3 grid((rows + 7) / 8), block(256);
    if (r.maxP <= 8) return launch_k(pkv::splitk_reduce_warp_kernel<T, D, 8, 8>, grid, block, 0, st, r);
    return launch_k(pkv::splitk_reduce_warp_kernel<T, D, 8, 0>, grid, block, 0, st, r);
}

constexpr int kMinMergePartition = 512;

// Split-K partials merged inside the decode kernel that supports it
// (pkv::merge_if_last) instead of by the reduce kernel; PKV_SPLIT_MERGE=0
// builds always run the reduce.
#ifndef PKV_SPLIT_MERGE
#define PKV_SPLIT_MERGE 1
#endif

// Longest-first unit order (pkv::lpt_unit) for at most 32 * kLptPerLane
// sequences and kLptMaxRanks ranks (sequences x partitions); the value is the
// sequences per lane (1, 2, 4 or 8), 0 for grid order.  Ranks without a unit
// come last in that order, each CTA of them deriving the order before it
// leaves: with many more ranks than units (a long max_context_len over short
// contexts) that tail costs more than the order saves, where grid order
// spreads the empty CTAs among the working ones.  PKV_LPT=0 builds keep grid
// order.
#ifndef PKV_LPT
#define PKV_LPT 1
#endif
constexpr int64_t kLptMaxRanks = 1024;
static int lpt_order(const pkv::AttnParams& p, int nparts) {
    if (!PKV_LPT || p.S > 32 * pkv::kLptPerLane || (int64_t)p.S * nparts > kLptMaxRanks) return 0;
    int per = 1;
    while (32 * per < p.S) per *= 2;
    return per;
}

// The per-sequence decode kernel of a call (no prefix pass, no reduce).
// *merged: the kernel merges the call's split-K partials itself (the MHA
// kernel with split counters), so no reduce kernel is to run.
template <typename T>
static cudaError_t decode_pass(const pkv::AttnParams& p, int D, int nparts, bool use_mma, const CUtensorMap* mk,
                               const CUtensorMap* mv, cudaStream_t st, bool* merged) {
    *merged = false;
    if constexpr (!std::is_same<T, float>::value) {
        if (use_mma) {
            dim3 grid((p.Hkv + kMmaWarps - 1) / kMmaWarps, nparts, p.S);
            return D == 64 ? launch_mma<T, 64>(p, grid, *mk, *mv, st) : launch_mma<T, 128>(p, grid, *mk, *mv, st);
        }
    }
    dim3 grid((p.Hq + kSimtWarps - 1) / kSimtWarps, nparts, p.S);
    pkv::AttnParams q = p;
    q.lpt = lpt_order(p, nparts);
    if (!PKV_SPLIT_MERGE) q.split_count = nullptr;
    *merged = q.split_count != nullptr;
    return D == 64 ? launch_simt<T, 64>(q, grid, st) : launch_simt<T, 128>(q, grid, st);
}

template <typename T>
static cudaError_t dispatch_attention(const pkv::AttnParams& p, int D, int nparts, int npre, bool use_mma,
                                      bool shared_mode, const CUtensorMap* mk, const CUtensorMap* mv,
                                      cudaStream_t st) {
    cudaError_t e = cudaSuccess;
    bool merged = false;  // the decode kernel merged the partials itself
    if constexpr (std::is_same<T, float>::value) {
        if (use_mma || shared_mode) return cudaErrorInvalidValue;
        e = decode_pass<T>(p, D, nparts, use_mma, mk, mv, st, &merged);
    } else {
        if (shared_mode && p.num_groups > 0) {  // membership first: every later kernel reads it
            e = launch_k(pkv::group_members_kernel, dim3((unsigned)((p.S + 7) / 8)), dim3(256), 0, st, p,
                         const_cast<int2*>(p.member));
            if (e != cudaSuccess) return e;
        }
        if (shared_mode && p.num_groups > 0 && npre > 0) {
            const int tiles = (p.max_group_size * p.G + 15) / 16;
            dim3 grid(tiles, npre, p.num_groups * p.Hkv);
            std::unique_lock<std::mutex> lk(g_side_mu);
            SideStream* ss = side_stream();
            cudaStream_t ps = st;
            if (ss != nullptr && cudaEventRecord(ss->fork, st) == cudaSuccess &&
                cudaStreamWaitEvent(ss->stream, ss->fork, 0) == cudaSuccess)
                ps = ss->stream;
            e = D == 64            ? launch_prefix<T, 64>(p, grid, *mk, *mv, ps)
                : PKV_PREFIX_TC != 0 ? launch_prefix_tc<T>(p, npre, *mk, *mv, ps)
                                     : launch_prefix<T, 128>(p, grid, *mk, *mv, ps);
            if (e == cudaSuccess) e = decode_pass<T>(p, D, nparts, use_mma, mk, mv, st, &merged);
            if (ps != st) {  // join, whatever happened above
                const cudaError_t j = cudaEventRecord(ss->join, ps);
                const cudaError_t w = j == cudaSuccess ? cudaStreamWaitEvent(st, ss->join, 0) : j;
                if (e == cudaSuccess) e = w;
            }
        } else {
            e = decode_pass<T>(p, D, nparts, use_mma, mk, mv, st, &merged);
        }
    }
    if (e != cudaSuccess || p.maxP <= 1 || merged) return e;
    pkv::ReduceParams r{p.out, p.ws_o, p.ws_ml, p.context_lens, p.S, p.Hq, D, p.P, p.maxP, p.max_len, p.bs,
                        p.member, nullptr, 0};
    return D == 64 ? launch_reduce<T, 64>(r, st) : launch_reduce<T, 128>(r, st);
}

// Per-head FP8 decode at head_dim 128 on tcgen05 (build-time switch).
#ifndef PKV_FP8_TC
#define PKV_FP8_TC 0
#endif
#ifndef PKV_FP8_TC_STAGES
#define PKV_FP8_TC_STAGES 2
#endif

template <typename To>
static cudaError_t launch_head_fp8_tc(const pkv::AttnParams& p, int nparts, const CUtensorMap& mk, const CUtensorMap& mv,
                                      cudaStream_t st) {
    using C = pkv::Fp8TcCfg<PKV_FP8_TC_STAGES>;
    auto k = pkv::paged_attn_fp8_tc_kernel<PKV_FP8_TC_STAGES, To>;
    static cudaError_t attr = set_smem(k, C::kSmemBytes);
    if (attr != cudaSuccess) return attr;
    return launch_k(k, dim3(p.Hq, nparts, p.S), dim3(128), C::kSmemBytes, st, p, mk, mv);
}

template <typename To>
static cudaError_t dispatch_attention_fp8(const pkv::AttnParams& p, int D, int nparts, bool use_mma,
                                          const CUtensorMap* mk, const CUtensorMap* mv, cudaStream_t st) {
    cudaError_t e;
    pkv::AttnParams q = p;  // the per-head kernel merges its own partials; the others leave them to the reduce
    if (use_mma) {
        q.split_count = nullptr;
        dim3 grid((p.Hkv + kMmaWarps - 1) / kMmaWarps, nparts, p.S);
        e = D == 64 ? launch_mma_fp8<To, 64>(q, grid, *mk, *mv, st) : launch_mma_fp8<To, 128>(q, grid, *mk, *mv, st);
    } else if (PKV_FP8_TC && D == 128) {
        q.split_count = nullptr;
        e = launch_head_fp8_tc<To>(q, nparts, *mk, *mv, st);
    } else {
        dim3 grid((p.Hq + kMmaWarps - 1) / kMmaWarps, nparts, p.S);
        q.lpt = lpt_order(p, nparts);
        if (!PKV_SPLIT_MERGE) q.split_count = nullptr;
        e = D == 64 ? launch_head_fp8<To, 64>(q, grid, *mk, *mv, st) : launch_head_fp8<To, 128>(q, grid, *mk, *mv, st);
    }
    if (e != cudaSuccess || p.maxP <= 1 || q.split_count != nullptr) return e;
    pkv::ReduceParams r{p.out, p.ws_o, p.ws_ml, p.context_lens, p.S, p.Hq, D, p.P, p.maxP, p.max_len, p.bs,
                        nullptr, nullptr, 0};
    return D == 64 ? launch_reduce<To, 64>(r, st) : launch_reduce<To, 128>(r, st);
}

// Built-in split-K scratch, for callers that cannot allocate.
//
// Some callers have no way to hand us device memory for the split-K
// workspace: code that runs where cudaMalloc is off limits (a host process
// whose allocator owns all device memory and forbids side allocations, a
// plug-in that may only use what it is given, code that must not reach a
// synchronising allocation in the middle of a step).  For them
// pkv_paged_attention_decode_static takes the partials from a fixed buffer
// compiled into this library.
//
// The buffer is one file-scope device array of kStaticScratchBytes per GPU,
// held by every GPU that loads this library until the process exits.  Its
// device address is looked up on each call that needs it (cudaGetSymbolAddress
// allocates nothing), with the calling device current, so a module reloaded
// at another address (a new context on the device) is always found; the
// host-side name of the array is not a device address and is never handed to
// a kernel.
constexpr size_t kStaticScratchBytes = size_t(64) << 20;  // 64 MiB per GPU
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

static cudaError_t static_scratch(void** ptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return e;
    *ptr = p;
    return cudaSuccess;
}

struct KvArgs {
    pkv_dtype dtype = PKV_BF16;  // pool element type (the call's type unless FP8)
    bool fp8 = false;
    float k_scale = 1.f, v_scale = 1.f;
};

struct GroupArgs {
    const int32_t* first = nullptr;
    const int32_t* shared = nullptr;
    int num = 0;
    int max_size = 0;
    int max_shared = 0;  // host bound on group_shared (sizes the prefix grid)
    bool mode = false;   // called through the shared-prefix entry point
};

static pkv_status decode_impl(void* out, const void* q, const void* k_pool, const void* v_pool,
                              const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
                              int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                              int num_blocks, float scale, int partition_size, const GroupArgs& grp, void* workspace,
                              size_t workspace_bytes, pkv_dtype dtype, void* stream, const KvArgs& kv = KvArgs(),
                              bool builtin_scratch = false) {
    if (!valid_dtype(dtype)) return invalid("pkv_paged_attention_decode: bad dtype");
    if (kv.fp8) {
        if (dtype == PKV_F32) {
            g_msg = "pkv_paged_attention_decode_fp8: q/out must be bf16 or f16";
            return PKV_ERR_UNSUPPORTED;
        }
        if (!(std::isfinite(kv.k_scale) && std::isfinite(kv.v_scale)) || kv.k_scale <= 0.f || kv.v_scale <= 0.f)
            return invalid("pkv_paged_attention_decode_fp8: k_scale and v_scale must be positive and finite");
        if (grp.mode) {
            g_msg = "pkv_paged_attention_decode_fp8: no shared-prefix mode for FP8 pools";
            return PKV_ERR_UNSUPPORTED;
        }
    }
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_blocks <= 0 || max_blocks_per_seq <= 0)
        return invalid("pkv_paged_attention_decode: sizes must be positive");
    if (num_q_heads > 65535) return invalid("pkv_paged_attention_decode: at most 65535 query heads");
    if (num_q_heads % num_kv_heads != 0)
        return invalid("pkv_paged_attention_decode: num_q_heads must be a multiple of num_kv_heads");
    if (!valid_block_size(block_size))
        return invalid("pkv_paged_attention_decode: block_size must be 16, 32, 64, 128 or 256");
    if (head_dim != 64 && head_dim != 128) {
        g_msg = "pkv_paged_attention_decode: head_dim must be 64 or 128";
        return PKV_ERR_UNSUPPORTED;
    }
    if (grp.mode && dtype == PKV_F32) {
        g_msg = "pkv_paged_attention_decode_shared: fp32 is not supported (tensor-core prefix pass)";
        return PKV_ERR_UNSUPPORTED;
    }
    if (partition_size < 0 || partition_size % 16 != 0)
        return invalid("pkv_paged_attention_decode: partition_size must be 0 or a positive multiple of 16");
    if (!(std::isfinite(scale)) || scale < 0.f) return invalid("pkv_paged_attention_decode: scale must be >= 0");
    const int64_t max_len64 = (int64_t)max_blocks_per_seq * block_size;
    if (max_len64 > (int64_t)1 << 30) return invalid("pkv_paged_attention_decode: max_blocks_per_seq*block_size too large");
    if ((int64_t)num_blocks * num_kv_heads * block_size >= ((int64_t)1 << 31))
        return invalid("pkv_paged_attention_decode: pool has 2^31 or more rows");
    if (grp.mode) {
        if (grp.num < 0) return invalid("pkv_paged_attention_decode_shared: num_groups must be >= 0");
        if (grp.num > 0 && (!grp.first || !grp.shared || (reinterpret_cast<uintptr_t>(grp.first) & 3u) ||
                            (reinterpret_cast<uintptr_t>(grp.shared) & 3u)))
            return invalid("pkv_paged_attention_decode_shared: group arrays must be 4-byte aligned device pointers");
        if (grp.num > 0 && grp.max_size < 1)
            return invalid("pkv_paged_attention_decode_shared: max_group_size must be >= 1");
        if ((int64_t)grp.num * num_kv_heads > 65535)
            return invalid("pkv_paged_attention_decode_shared: num_groups * num_kv_heads must be <= 65535");
        if ((int64_t)grp.max_size * (num_q_heads / num_kv_heads) > ((int64_t)1 << 24))
            return invalid("pkv_paged_attention_decode_shared: max_group_size too large");
        if (grp.num > 0 && (grp.max_shared < 0 || grp.max_shared > max_len64))
            return invalid("pkv_paged_attention_decode_shared: max_shared_len must be in [0, max_blocks_per_seq*block_size]");
    }
    if (num_seqs == 0) return PKV_OK;
    if (!out || !q || !k_pool || !v_pool || !block_tables || !context_lens)
        return invalid("pkv_paged_attention_decode: null pointer");
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) ||
        (reinterpret_cast<uintptr_t>(block_tables) & 3u) || (reinterpret_cast<uintptr_t>(context_lens) & 3u))
        return invalid("pkv_paged_attention_decode: pointers must be 16-byte aligned (tables 4-byte)");
    if (num_seqs > 65535) return invalid("pkv_paged_attention_decode: at most 65535 sequences per call");

    const int max_len = (int)max_len64;
    const int P = choose_partition(max_len, partition_size);
    const int64_t nparts = (max_len + P - 1) / P;
    if (nparts > 65535) return invalid("pkv_paged_attention_decode: too many partitions; raise partition_size");
    const int64_t slots = nparts + (grp.mode ? 1 : 0);
    const size_t need = grp.mode ? shared_workspace_for(num_seqs, num_q_heads, head_dim, max_len, P)
                                 : workspace_for(num_seqs, num_q_heads, head_dim, max_len, P);
    if (need > 0 && builtin_scratch) {  // every other argument has passed by now
        if (need > kStaticScratchBytes) {
            g_msg = "pkv_paged_attention_decode_static: this call needs " + std::to_string(need) +
                    " bytes of split-K scratch but the built-in buffer holds " + std::to_string(kStaticScratchBytes) +
                    "; use a larger partition_size, fewer sequences, or pkv_paged_attention_decode with a "
                    "caller-provided workspace";
            return PKV_ERR_INVALID;
        }
        const cudaError_t e = static_scratch(&workspace);
        if (e != cudaSuccess) return cuda_fail("pkv_paged_attention_decode_static: scratch address", e);
        workspace_bytes = kStaticScratchBytes;
    }
    if (need > 0) {
        if (!workspace || workspace_bytes < need) return invalid("pkv_paged_attention_decode: workspace too small");
        if (reinterpret_cast<uintptr_t>(workspace) & 255u)
            return invalid("pkv_paged_attention_decode: workspace must be 256-byte aligned");
    }

    pkv::AttnParams p;
    std::memset(&p, 0, sizeof p);
    p.out = out;
    p.q = q;
    p.k_pool = k_pool;
    p.v_pool = v_pool;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    const size_t n_part = (size_t)num_seqs * num_q_heads * slots;
    p.ws_o = need ? static_cast<float*>(workspace) : nullptr;
    p.ws_ml = need ? static_cast<float*>(workspace) + n_part * head_dim : nullptr;
    p.S = num_seqs;
    p.Hq = num_q_heads;
    p.Hkv = num_kv_heads;
    p.G = num_q_heads / num_kv_heads;
    p.bs = block_size;
    p.NB = num_blocks;
    p.maxB = max_blocks_per_seq;
    p.P = P;
    p.maxP = (int)slots;
    p.max_len = max_len;
    const float sc = scale > 0.f ? scale : 1.f / std::sqrt((float)head_dim);
    p.scale_log2 = sc * 1.4426950408889634f * (kv.fp8 ? kv.k_scale : 1.f);
    p.v_scale = kv.fp8 ? kv.v_scale : 1.f;
    p.group_first = grp.num > 0 ? grp.first : nullptr;
    p.group_shared = grp.num > 0 ? grp.shared : nullptr;
    p.num_groups = grp.num;
    p.max_group_size = grp.max_size;
    p.max_shared = grp.max_shared;
    // Shared-prefix membership after the partials (8-byte aligned: (D+2)*4 is).
    p.member = grp.mode && grp.num > 0 ? reinterpret_cast<const int2*>(p.ws_ml + n_part * 2) : nullptr;
    // Split counters (their own region of the workspace without groups); a
    // kernel that cannot merge its own partials gets nullptr and the reduce
    // runs.  The merge costs each CTA a fence and an exchange at its end,
    // repaid only by long units: from 512-token partitions on (shorter ones
    // measured 2-4 % slower than the reduce kernel).
    if (need > 0 && !grp.mode && slots <= 32 && P >= kMinMergePartition) {
        p.split_count = reinterpret_cast<unsigned long long*>(
            static_cast<char*>(workspace) + split_counters_offset(partials_bytes((int64_t)num_seqs * num_q_heads,
                                                                                 slots, head_dim)));
        p.stamp = next_call_stamp();
    }

    const bool use_mma = dtype != PKV_F32 && p.G >= 2 && p.G <= 16;
    CUtensorMap mk, mv;
    if (kv.fp8) {  // both FP8 kernels read 16-token boxes of codes
        const int64_t rows = (int64_t)num_blocks * num_kv_heads * block_size;
        if (!make_pool_map(&mk, k_pool, rows, head_dim, PKV_FP8_E4M3, head_dim == 128) ||
            !make_pool_map(&mv, v_pool, rows, head_dim, PKV_FP8_E4M3, head_dim == 128)) {
            g_msg = "pkv_paged_attention_decode_fp8: cuTensorMapEncodeTiled failed";
            return PKV_ERR_CUDA;
        }
        cudaError_t e = dtype == PKV_BF16
                            ? dispatch_attention_fp8<__nv_bfloat16>(p, head_dim, (int)nparts, use_mma, &mk, &mv,
                                                                    (cudaStream_t)stream)
                            : dispatch_attention_fp8<__half>(p, head_dim, (int)nparts, use_mma, &mk, &mv,
                                                             (cudaStream_t)stream);
        return e == cudaSuccess ? PKV_OK : cuda_fail("pkv_paged_attention_decode_fp8", e);
    }
    if (use_mma || (grp.mode && grp.num > 0)) {
        const int64_t rows = (int64_t)num_blocks * num_kv_heads * block_size;
        if (!make_pool_map(&mk, k_pool, rows, head_dim, dtype, true) || !make_pool_map(&mv, v_pool, rows, head_dim, dtype, true)) {
            g_msg = "pkv_paged_attention_decode: cuTensorMapEncodeTiled failed";
            return PKV_ERR_CUDA;
        }
    }
    cudaStream_t st = (cudaStream_t)stream;
    const int npre = (grp.max_shared + P - 1) / P;  // partitions of the longest shared run
    cudaError_t e;
    switch (dtype) {
        case PKV_F32:
            e = dispatch_attention<float>(p, head_dim, (int)nparts, 0, false, false, nullptr, nullptr, st);
            break;
        case PKV_BF16:
            e = dispatch_attention<__nv_bfloat16>(p, head_dim, (int)nparts, npre, use_mma, grp.mode, &mk, &mv, st);
            break;
        default:
            e = dispatch_attention<__half>(p, head_dim, (int)nparts, npre, use_mma, grp.mode, &mk, &mv, st);
            break;
    }
    return e == cudaSuccess ? PKV_OK : cuda_fail("pkv_paged_attention_decode", e);
}

}  // namespace pkv_host

using namespace pkv_host;

extern "C" {

const char* pkv_status_str(pkv_status s) {
    switch (s) {
        case PKV_OK: return "ok";
        case PKV_ERR_INVALID: return "invalid argument";
        case PKV_ERR_NO_FREE_BLOCK: return "no free block";
        case PKV_ERR_CUDA: return "CUDA error";
        case PKV_ERR_UNSUPPORTED: return "unsupported configuration";
        case PKV_ERR_DEVICE_CHECK: return "device-side index check failed";
    }
    return "unknown status";
}

const char* pkv_last_error(void) { return g_msg.c_str(); }

uint64_t pkv_launch_count(void) { return g_launches.load(); }

pkv_status pkv_kv_append(const void* k_new, const void* v_new, void* k_pool, void* v_pool,
                         const int64_t* slot_mapping, int num_tokens, int num_blocks, int num_kv_heads,
                         int head_dim, int block_size, pkv_dtype dtype, void* stream) {
    if (!valid_dtype(dtype)) return invalid("pkv_kv_append: bad dtype");
    if (num_tokens < 0 || num_blocks <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0)
        return invalid("pkv_kv_append: sizes must be positive");
    const int row_bytes = head_dim * elem_size(dtype);
    if (row_bytes % 16 != 0) return invalid("pkv_kv_append: head_dim * element size must be a multiple of 16 bytes");
    if (num_tokens == 0) return PKV_OK;
    if (!k_new || !v_new || !k_pool || !v_pool || !slot_mapping)
        return invalid("pkv_kv_append: null pointer");
    if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_pool) || !aligned16(v_pool) ||
        (reinterpret_cast<uintptr_t>(slot_mapping) & 7u))
        return invalid("pkv_kv_append: pointers must be 16-byte aligned (slot_mapping 8-byte)");
    pkv::AppendParams p;
    p.k_new = static_cast<const uint4*>(k_new);
    p.v_new = static_cast<const uint4*>(v_new);
    p.k_pool = static_cast<uint4*>(k_pool);
    p.v_pool = static_cast<uint4*>(v_pool);
    p.slot_mapping = slot_mapping;
    p.vecs_per_row = row_bytes / 16;
    p.Hkv = num_kv_heads;
    p.bs = block_size;
    p.num_slots = (int64_t)num_blocks * block_size;
    p.total_vecs = (int64_t)num_tokens * num_kv_heads * p.vecs_per_row;
    int64_t blocks = (p.total_vecs + 255) / 256;
    const int64_t cap = (int64_t)num_sms() * 16;
    if (blocks > cap) blocks = cap;
    cudaError_t e = launch_k(pkv::kv_append_kernel, dim3((unsigned)blocks), dim3(256), 0, (cudaStream_t)stream, p);
    return e == cudaSuccess ? PKV_OK : cuda_fail("pkv_kv_append", e);
}

size_t pkv_attention_workspace_bytes(int num_seqs, int num_q_heads, int head_dim, int max_context_len,
                                     int partition_size) {
    if (num_seqs <= 0 || num_q_heads <= 0 || head_dim <= 0 || max_context_len <= 0 || partition_size < 0) return 0;
    return workspace_for(num_seqs, num_q_heads, head_dim, max_context_len,
                         partition_bound(max_context_len, partition_size));
}

int pkv_attention_partition_size(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int max_context_len,
                                 int partition_size) {
    (void)num_seqs;
    (void)num_q_heads;
    (void)num_kv_heads;
    (void)head_dim;
    return choose_partition(max_context_len, partition_size);
}

pkv_status pkv_paged_attention_decode(void* out, const void* q, const void* k_pool, const void* v_pool,
                                      const int32_t* block_tables, int max_blocks_per_seq,
                                      const int32_t* context_lens, int num_seqs, int num_q_heads, int num_kv_heads,
                                      int head_dim, int block_size, int num_blocks, float scale, int partition_size,
                                      void* workspace, size_t workspace_bytes, pkv_dtype dtype, void* stream) {
    return decode_impl(out, q, k_pool, v_pool, block_tables, max_blocks_per_seq, context_lens, num_seqs, num_q_heads,
                       num_kv_heads, head_dim, block_size, num_blocks, scale, partition_size, GroupArgs(), workspace,
                       workspace_bytes, dtype, stream);
}

pkv_status pkv_paged_attention_decode_shared(void* out, const void* q, const void* k_pool, const void* v_pool,
                                             const int32_t* block_tables, int max_blocks_per_seq,
                                             const int32_t* context_lens, int num_seqs, int num_q_heads,
                                             int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                             float scale, int partition_size, const int32_t* group_first,
                                             const int32_t* group_shared, int num_groups, int max_group_size,
                                             int max_shared_len, void* workspace, size_t workspace_bytes,
                                             pkv_dtype dtype, void* stream) {
    GroupArgs g;
    g.first = group_first;
    g.shared = group_shared;
    g.num = num_groups;
    g.max_size = max_group_size;
    g.max_shared = max_shared_len;
    g.mode = true;
    return decode_impl(out, q, k_pool, v_pool, block_tables, max_blocks_per_seq, context_lens, num_seqs, num_q_heads,
                       num_kv_heads, head_dim, block_size, num_blocks, scale, partition_size, g, workspace,
                       workspace_bytes, dtype, stream);
}

size_t pkv_attention_shared_workspace_bytes(int num_seqs, int num_q_heads, int head_dim, int max_context_len,
                                            int partition_size) {
    if (num_seqs <= 0 || num_q_heads <= 0 || head_dim <= 0 || max_context_len <= 0 || partition_size < 0) return 0;
    return shared_workspace_for(num_seqs, num_q_heads, head_dim, max_context_len,
                                partition_bound(max_context_len, partition_size));
}

pkv_status pkv_block_copy(void* k_pool, void* v_pool, const int32_t* pairs, int num_pairs, int num_blocks,
                          int num_kv_heads, int head_dim, int block_size, pkv_dtype dtype, void* stream) {
    if (!valid_dtype(dtype) && dtype != PKV_FP8_E4M3) return invalid("pkv_block_copy: bad dtype");
    if (num_pairs < 0 || num_blocks <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0)
        return invalid("pkv_block_copy: sizes must be positive");
    const int64_t block_bytes = (int64_t)num_kv_heads * block_size * head_dim * elem_size(dtype);
    if (block_bytes % 16 != 0) return invalid("pkv_block_copy: block bytes must be a multiple of 16");
    if (num_pairs == 0) return PKV_OK;
    if (!k_pool || !v_pool || !pairs) return invalid("pkv_block_copy: null pointer");
    if (!aligned16(k_pool) || !aligned16(v_pool) || (reinterpret_cast<uintptr_t>(pairs) & 3u))
        return invalid("pkv_block_copy: pools must be 16-byte aligned");
    pkv::CopyParams p;
    p.k_pool = static_cast<uint4*>(k_pool);
    p.v_pool = static_cast<uint4*>(v_pool);
    p.pairs = pairs;
    p.block_vecs = block_bytes / 16;
    p.num_blocks = num_blocks;
    // ~4 vectors of K and of V per thread, at most 64 slices per block.
    int64_t slices = (p.block_vecs + 1023) / 1024;
    if (slices > 64) slices = 64;
    if (num_pairs > 2147483647) return invalid("pkv_block_copy: too many pairs");
    cudaError_t e = launch_k(pkv::block_copy_kernel, dim3((unsigned)num_pairs, (unsigned)slices), dim3(256), 0,
                             (cudaStream_t)stream, p);
    return e == cudaSuccess ? PKV_OK : cuda_fail("pkv_block_copy", e);
}

pkv_status pkv_device_error(void* stream, uint32_t* code) {
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail("pkv_device_error: stream", e);
    unsigned int v = 0;
    e = cudaMemcpyFromSymbol(&v, pkv::g_device_error, sizeof v);
    if (e != cudaSuccess) return cuda_fail("pkv_device_error: read", e);
    if (v) {
        unsigned int zero = 0;
        e = cudaMemcpyToSymbol(pkv::g_device_error, &zero, sizeof zero);
        if (e != cudaSuccess) return cuda_fail("pkv_device_error: clear", e);
    }
    if (code) *code = v;
    if (v) {
        g_msg = "device-side index check recorded bits " + std::to_string(v);
        return PKV_ERR_DEVICE_CHECK;
    }
    return PKV_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// FP8 E4M3 pools.
// ---------------------------------------------------------------------------
extern "C" pkv_status pkv_kv_append_fp8(const void* k_new, const void* v_new, void* k_pool, void* v_pool,
                                        const int64_t* slot_mapping, int num_tokens, int num_blocks,
                                        int num_kv_heads, int head_dim, int block_size, pkv_dtype src_dtype,
                                        float k_scale, float v_scale, void* stream) {
    using namespace pkv_host;
    if (src_dtype != PKV_F32 && src_dtype != PKV_BF16 && src_dtype != PKV_F16)
        return invalid("pkv_kv_append_fp8: new K/V must be f32, bf16 or f16");
    if (num_tokens < 0 || num_blocks <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0)
        return invalid("pkv_kv_append_fp8: sizes must be positive");
    if (head_dim % 16 != 0) return invalid("pkv_kv_append_fp8: head_dim must be a multiple of 16");
    if (!(std::isfinite(k_scale) && std::isfinite(v_scale)) || k_scale <= 0.f || v_scale <= 0.f)
        return invalid("pkv_kv_append_fp8: k_scale and v_scale must be positive and finite");
    if (num_tokens == 0) return PKV_OK;
    if (!k_new || !v_new || !k_pool || !v_pool || !slot_mapping) return invalid("pkv_kv_append_fp8: null pointer");
    if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_pool) || !aligned16(v_pool) ||
        (reinterpret_cast<uintptr_t>(slot_mapping) & 7u))
        return invalid("pkv_kv_append_fp8: pointers must be 16-byte aligned (slot_mapping 8-byte)");
    pkv::AppendFp8Params p;
    p.k_new = k_new;
    p.v_new = v_new;
    p.k_pool = static_cast<uint4*>(k_pool);
    p.v_pool = static_cast<uint4*>(v_pool);
    p.slot_mapping = slot_mapping;
    p.vecs_per_row = head_dim / 16;
    p.Hkv = num_kv_heads;
    p.bs = block_size;
    p.num_slots = (int64_t)num_blocks * block_size;
    p.total_vecs = (int64_t)num_tokens * num_kv_heads * p.vecs_per_row;
    p.k_inv = 1.0f / k_scale;  // the inverse is rounded to fp32 once, on the host
    p.v_inv = 1.0f / v_scale;
    int64_t blocks = (p.total_vecs + 255) / 256;
    const int64_t cap = (int64_t)num_sms() * 16;
    if (blocks > cap) blocks = cap;
    cudaStream_t st = (cudaStream_t)stream;
    const dim3 grid((unsigned)blocks), block(256);
    cudaError_t e = src_dtype == PKV_F32    ? launch_k(pkv::kv_append_fp8_kernel<float>, grid, block, 0, st, p)
                    : src_dtype == PKV_BF16 ? launch_k(pkv::kv_append_fp8_kernel<__nv_bfloat16>, grid, block, 0, st, p)
                                            : launch_k(pkv::kv_append_fp8_kernel<__half>, grid, block, 0, st, p);
    return e == cudaSuccess ? PKV_OK : cuda_fail("pkv_kv_append_fp8", e);
}

extern "C" pkv_status pkv_paged_attention_decode_fp8(void* out, const void* q, const void* k_pool,
                                                     const void* v_pool, const int32_t* block_tables,
                                                     int max_blocks_per_seq, const int32_t* context_lens,
                                                     int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                                     int block_size, int num_blocks, float scale, float k_scale,
                                                     float v_scale, int partition_size, void* workspace,
                                                     size_t workspace_bytes, pkv_dtype dtype, void* stream) {
    using namespace pkv_host;
    KvArgs kv;
    kv.dtype = PKV_FP8_E4M3;
    kv.fp8 = true;
    kv.k_scale = k_scale;
    kv.v_scale = v_scale;
    return decode_impl(out, q, k_pool, v_pool, block_tables, max_blocks_per_seq, context_lens, num_seqs, num_q_heads,
                       num_kv_heads, head_dim, block_size, num_blocks, scale, partition_size, GroupArgs(), workspace,
                       workspace_bytes, dtype, stream, kv);
}

// ---------------------------------------------------------------------------
// Causal attention for a chunk of new tokens per sequence.
// ---------------------------------------------------------------------------
namespace pkv_host {

static size_t chunk_workspace_for(int T, int Hq, int D, int max_len, int P) {
    const int64_t nparts = ((int64_t)max_len + P - 1) / P;
    if (nparts <= 1) return 0;
    return partials_bytes((int64_t)T * Hq, nparts, D);
}

template <typename T>
static cudaError_t dispatch_chunk(const pkv::AttnParams& p, const pkv::ChunkParams& c, int D, int tiles,
                                  const CUtensorMap& mk, const CUtensorMap& mv, cudaStream_t st) {
    if constexpr (std::is_same<T, float>::value) {
        return cudaErrorInvalidValue;
    } else {
        dim3 grid((p.Hkv + kMmaWarps - 1) / kMmaWarps, tiles * c.nparts, p.S);
        cudaError_t e = D == 64 ? launch_chunk<T, 64>(p, c, grid, mk, mv, st) : launch_chunk<T, 128>(p, c, grid, mk, mv, st);
        if (e != cudaSuccess || c.nparts <= 1) return e;
        pkv::ReduceParams r{p.out, p.ws_o, p.ws_ml, p.context_lens, p.S, p.Hq, D, p.P, p.maxP, p.max_len, p.bs,
                            nullptr, c.query_start, c.T};
        return D == 64 ? launch_reduce<T, 64>(r, st) : launch_reduce<T, 128>(r, st);
    }
}

}  // namespace pkv_host

extern "C" size_t pkv_attention_chunk_workspace_bytes(int num_tokens, int num_q_heads, int head_dim,
                                                      int max_context_len, int partition_size) {
    using namespace pkv_host;
    if (num_tokens <= 0 || num_q_heads <= 0 || head_dim <= 0 || max_context_len <= 0 || partition_size < 0) return 0;
    return chunk_workspace_for(num_tokens, num_q_heads, head_dim, max_context_len,
                               partition_bound(max_context_len, partition_size));
}

extern "C" pkv_status pkv_paged_attention_chunk(void* out, const void* q, const void* k_pool, const void* v_pool,
                                                const int32_t* block_tables, int max_blocks_per_seq,
                                                const int32_t* context_lens, const int32_t* query_start,
                                                int num_seqs, int num_tokens, int max_query_len, int num_q_heads,
                                                int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                                float scale, int partition_size, void* workspace,
                                                size_t workspace_bytes, pkv_dtype dtype, void* stream) {
    using namespace pkv_host;
    const char* fn = "pkv_paged_attention_chunk";
    if (dtype != PKV_BF16 && dtype != PKV_F16) {
        g_msg = std::string(fn) + ": 16-bit element types only (tensor-core kernel)";
        return valid_dtype(dtype) ? PKV_ERR_UNSUPPORTED : PKV_ERR_INVALID;
    }
    if (num_seqs < 0 || num_tokens < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_blocks <= 0 ||
        max_blocks_per_seq <= 0 || max_query_len < 1)
        return invalid("pkv_paged_attention_chunk: sizes must be positive");
    if (num_q_heads > 65535) return invalid("pkv_paged_attention_chunk: at most 65535 query heads");
    if (num_q_heads % num_kv_heads != 0 || num_q_heads / num_kv_heads > 16)
        return invalid("pkv_paged_attention_chunk: num_q_heads must be 1..16 times num_kv_heads");
    if (!valid_block_size(block_size))
        return invalid("pkv_paged_attention_chunk: block_size must be 16, 32, 64, 128 or 256");
    if (head_dim != 64 && head_dim != 128) {
        g_msg = std::string(fn) + ": head_dim must be 64 or 128";
        return PKV_ERR_UNSUPPORTED;
    }
    if (partition_size < 0 || partition_size % 16 != 0)
        return invalid("pkv_paged_attention_chunk: partition_size must be 0 or a positive multiple of 16");
    if (!(std::isfinite(scale)) || scale < 0.f) return invalid("pkv_paged_attention_chunk: scale must be >= 0");
    const int64_t max_len64 = (int64_t)max_blocks_per_seq * block_size;
    if (max_len64 > (int64_t)1 << 30) return invalid("pkv_paged_attention_chunk: max_blocks_per_seq*block_size too large");
    if ((int64_t)num_blocks * num_kv_heads * block_size >= ((int64_t)1 << 31))
        return invalid("pkv_paged_attention_chunk: pool has 2^31 or more rows");
    if (num_seqs == 0 || num_tokens == 0) return PKV_OK;
    if (!out || !q || !k_pool || !v_pool || !block_tables || !context_lens || !query_start)
        return invalid("pkv_paged_attention_chunk: null pointer");
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) ||
        (reinterpret_cast<uintptr_t>(block_tables) & 3u) || (reinterpret_cast<uintptr_t>(context_lens) & 3u) ||
        (reinterpret_cast<uintptr_t>(query_start) & 3u))
        return invalid("pkv_paged_attention_chunk: pointers must be 16-byte aligned (int arrays 4-byte)");
    if (num_seqs > 65535) return invalid("pkv_paged_attention_chunk: at most 65535 sequences per call");
    const int max_len = (int)max_len64;
    const int G = num_q_heads / num_kv_heads;
    const int P = choose_partition(max_len, partition_size);
    const int64_t nparts = (max_len + P - 1) / P;
    const int64_t tiles = ((int64_t)max_query_len * G + 15) / 16;
    if (tiles * nparts > 65535) return invalid("pkv_paged_attention_chunk: too many row tiles x partitions");
    if ((int64_t)num_tokens * num_q_heads > INT32_MAX) return invalid("pkv_paged_attention_chunk: too many rows");
    const size_t need = chunk_workspace_for(num_tokens, num_q_heads, head_dim, max_len, P);
    if (need > 0) {
        if (!workspace || workspace_bytes < need) return invalid("pkv_paged_attention_chunk: workspace too small");
        if (reinterpret_cast<uintptr_t>(workspace) & 255u)
            return invalid("pkv_paged_attention_chunk: workspace must be 256-byte aligned");
    }
    pkv::AttnParams p;
    std::memset(&p, 0, sizeof p);
    p.out = out;
    p.q = q;
    p.k_pool = k_pool;
    p.v_pool = v_pool;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    const size_t n_part = (size_t)num_tokens * num_q_heads * nparts;
    p.ws_o = need ? static_cast<float*>(workspace) : nullptr;
    p.ws_ml = need ? static_cast<float*>(workspace) + n_part * head_dim : nullptr;
    p.S = num_seqs;
    p.Hq = num_q_heads;
    p.Hkv = num_kv_heads;
    p.G = G;
    p.bs = block_size;
    p.NB = num_blocks;
    p.maxB = max_blocks_per_seq;
    p.P = P;
    p.maxP = (int)nparts;
    p.max_len = max_len;
    const float sc = scale > 0.f ? scale : 1.f / std::sqrt((float)head_dim);
    p.scale_log2 = sc * 1.4426950408889634f;
    p.v_scale = 1.f;
    pkv::ChunkParams c{query_start, num_tokens, max_query_len, (int)nparts};
    CUtensorMap mk, mv;
    const int64_t rows = (int64_t)num_blocks * num_kv_heads * block_size;
    if (!make_pool_map(&mk, k_pool, rows, head_dim, dtype, true) || !make_pool_map(&mv, v_pool, rows, head_dim, dtype, true)) {
        g_msg = std::string(fn) + ": cuTensorMapEncodeTiled failed";
        return PKV_ERR_CUDA;
    }
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = dtype == PKV_BF16 ? dispatch_chunk<__nv_bfloat16>(p, c, head_dim, (int)tiles, mk, mv, st)
                                      : dispatch_chunk<__half>(p, c, head_dim, (int)tiles, mk, mv, st);
    return e == cudaSuccess ? PKV_OK : cuda_fail(fn, e);
}

extern "C" pkv_status pkv_paged_attention_decode_static(void* out, const void* q, const void* k_pool,
                                                        const void* v_pool, const int32_t* block_tables,
                                                        int max_blocks_per_seq, const int32_t* context_lens,
                                                        int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                                        int block_size, int num_blocks, float scale,
                                                        int partition_size, pkv_dtype dtype, void* stream) {
    using namespace pkv_host;
    return decode_impl(out, q, k_pool, v_pool, block_tables, max_blocks_per_seq, context_lens, num_seqs, num_q_heads,
                       num_kv_heads, head_dim, block_size, num_blocks, scale, partition_size, GroupArgs(), nullptr, 0,
                       dtype, stream, KvArgs(), true);
}

// ---------------------------------------------------------------------------
// A whole step from host buffers in one call: copies in, block_copy,
// kv_append, attention, copies out -- each part the same code as its own
// entry point, on one stream.
// ---------------------------------------------------------------------------
namespace pkv_host {

static pkv_status copies(const pkv_copy* c, int n, cudaStream_t st, const char* what) {
    for (int i = 0; i < n; ++i) {
        if (c[i].bytes == 0) continue;
        if (!c[i].dst || !c[i].src) {
            g_msg = std::string("pkv_step_from_host: null pointer in the ") + what + " copies";
            return PKV_ERR_INVALID;
        }
        const cudaError_t e = cudaMemcpyAsync(c[i].dst, c[i].src, c[i].bytes, cudaMemcpyDefault, st);
        if (e != cudaSuccess) return cuda_fail("pkv_step_from_host: copy", e);
    }
    return PKV_OK;
}

}  // namespace pkv_host

extern "C" pkv_status pkv_step_from_host(const pkv_step* s, void* stream) {
    using namespace pkv_host;
    if (!s) return invalid("pkv_step_from_host: null step");
    if (s->struct_size != sizeof(pkv_step))
        return invalid("pkv_step_from_host: struct_size is not sizeof(pkv_step) (header version mismatch)");
    if (s->kind < PKV_STEP_DECODE || s->kind > PKV_STEP_CHUNK) return invalid("pkv_step_from_host: bad kind");
    if (s->n_in < 0 || s->n_out < 0 || (s->n_in > 0 && !s->in) || (s->n_out > 0 && !s->out))
        return invalid("pkv_step_from_host: bad copy lists");
    if (s->num_pairs < 0 || s->num_tokens < 0 || s->num_seqs < 0)
        return invalid("pkv_step_from_host: counts must be >= 0");
    const bool split = s->copy_stream != nullptr;
    if (split != (s->inputs_free != nullptr) || split != (s->inputs_ready != nullptr))
        return invalid("pkv_step_from_host: copy_stream, inputs_free and inputs_ready go together");
    const bool split_out = s->out_stream != nullptr;
    if (split_out != (s->outputs_done != nullptr))
        return invalid("pkv_step_from_host: out_stream and outputs_done go together");
    if (split_out && !split)
        return invalid("pkv_step_from_host: out_stream needs copy_stream, inputs_free and inputs_ready");
    cudaStream_t st = (cudaStream_t)stream;
    const pkv_dtype dt = (pkv_dtype)s->dtype;
    const bool fp8 = s->kind == PKV_STEP_DECODE_FP8;
    pkv_status r;
    if (split) {  // the input copies on copy_stream, after the last reader of their destinations
        cudaStream_t cs = (cudaStream_t)s->copy_stream;
        cudaError_t e = cudaStreamWaitEvent(cs, (cudaEvent_t)s->inputs_free, 0);
        if (e != cudaSuccess) return cuda_fail("pkv_step_from_host: wait for inputs_free", e);
        r = copies(s->in, s->n_in, cs, "input");
        if (r != PKV_OK) return r;
        e = cudaEventRecord((cudaEvent_t)s->inputs_ready, cs);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(st, (cudaEvent_t)s->inputs_ready, 0);
        if (e != cudaSuccess) return cuda_fail("pkv_step_from_host: inputs_ready", e);
    } else {
        r = copies(s->in, s->n_in, st, "input");
        if (r != PKV_OK) return r;
    }
    if (s->num_pairs > 0) {
        r = pkv_block_copy(s->k_pool, s->v_pool, s->pairs, s->num_pairs, s->num_blocks, s->num_kv_heads,
                           s->head_dim, s->block_size, fp8 ? PKV_FP8_E4M3 : dt, stream);
        if (r != PKV_OK) return r;
    }
    if (s->num_tokens > 0) {
        r = fp8 ? pkv_kv_append_fp8(s->k_new, s->v_new, s->k_pool, s->v_pool, s->slot_mapping, s->num_tokens,
                                    s->num_blocks, s->num_kv_heads, s->head_dim, s->block_size, dt, s->k_scale,
                                    s->v_scale, stream)
                : pkv_kv_append(s->k_new, s->v_new, s->k_pool, s->v_pool, s->slot_mapping, s->num_tokens,
                                s->num_blocks, s->num_kv_heads, s->head_dim, s->block_size, dt, stream);
        if (r != PKV_OK) return r;
    }
    if (split_out) {  // the previous output copies out of attn_out have finished
        const cudaError_t e = cudaStreamWaitEvent(st, (cudaEvent_t)s->outputs_done, 0);
        if (e != cudaSuccess) return cuda_fail("pkv_step_from_host: wait for outputs_done", e);
    }
    if (s->num_seqs > 0) {
        switch (s->kind) {
            case PKV_STEP_DECODE:
                r = pkv_paged_attention_decode(s->attn_out, s->q, s->k_pool, s->v_pool, s->block_tables,
                                               s->max_blocks_per_seq, s->context_lens, s->num_seqs, s->num_q_heads,
                                               s->num_kv_heads, s->head_dim, s->block_size, s->num_blocks, s->scale,
                                               s->partition_size, s->workspace, s->workspace_bytes, dt, stream);
                break;
            case PKV_STEP_DECODE_SHARED:
                r = pkv_paged_attention_decode_shared(
                    s->attn_out, s->q, s->k_pool, s->v_pool, s->block_tables, s->max_blocks_per_seq, s->context_lens,
                    s->num_seqs, s->num_q_heads, s->num_kv_heads, s->head_dim, s->block_size, s->num_blocks,
                    s->scale, s->partition_size, s->group_first, s->group_shared, s->num_groups, s->max_group_size,
                    s->max_shared_len, s->workspace, s->workspace_bytes, dt, stream);
                break;
            case PKV_STEP_DECODE_FP8:
                r = pkv_paged_attention_decode_fp8(s->attn_out, s->q, s->k_pool, s->v_pool, s->block_tables,
                                                   s->max_blocks_per_seq, s->context_lens, s->num_seqs,
                                                   s->num_q_heads, s->num_kv_heads, s->head_dim, s->block_size,
                                                   s->num_blocks, s->scale, s->k_scale, s->v_scale,
                                                   s->partition_size, s->workspace, s->workspace_bytes, dt, stream);
                break;
            default:
                r = pkv_paged_attention_chunk(s->attn_out, s->q, s->k_pool, s->v_pool, s->block_tables,
                                              s->max_blocks_per_seq, s->context_lens, s->query_start, s->num_seqs,
                                              s->num_tokens, s->max_query_len, s->num_q_heads, s->num_kv_heads,
                                              s->head_dim, s->block_size, s->num_blocks, s->scale, s->partition_size,
                                              s->workspace, s->workspace_bytes, dt, stream);
                break;
        }
        if (r != PKV_OK) return r;
    }
    if (split) {  // nothing of this step reads the input copies' destinations after this point
        const cudaError_t e = cudaEventRecord((cudaEvent_t)s->inputs_free, st);
        if (e != cudaSuccess) return cuda_fail("pkv_step_from_host: inputs_free", e);
    }
    if (!split_out) return copies(s->out, s->n_out, st, "output");
    cudaStream_t os = (cudaStream_t)s->out_stream;  // the output copies after the kernels, off `stream`
    cudaError_t e = cudaStreamWaitEvent(os, (cudaEvent_t)s->inputs_free, 0);
    if (e != cudaSuccess) return cuda_fail("pkv_step_from_host: out_stream wait", e);
    r = copies(s->out, s->n_out, os, "output");
    if (r != PKV_OK) return r;
    e = cudaEventRecord((cudaEvent_t)s->outputs_done, os);
    return e == cudaSuccess ? PKV_OK : cuda_fail("pkv_step_from_host: outputs_done", e);
}
