// Pieces shared by the two paged decode attention kernels.
#pragma once
#include "common.cuh"

namespace pkv {

constexpr int kTileTok = 16;  // tokens per pipeline stage (block_size is a multiple)

struct AttnParams {
    void* out;                 // [S][Hq][D] of T
    const void* q;             // [S][Hq][D] of T
    const void* k_pool;        // [NB][Hkv][bs][D] of T
    const void* v_pool;
    const int32_t* block_tables;  // [S][maxB]
    const int32_t* context_lens;  // [S]
    float* ws_o;               // [S][Hq][maxP][D]   (split-K partials)
    float* ws_ml;              // [S][Hq][maxP][2]   (m, l) per partial
    int S, Hq, Hkv, G, bs, NB, maxB, P, maxP, max_len;
    float scale_log2;          // softmax scale * log2(e) (* k_scale for FP8 pools)
    float v_scale;             // V code scale for FP8 pools (1 otherwise), applied to outputs
    // Shared-prefix groups (num_groups = 0: none).  Group i is the sequences
    // group_first[i] .. group_first[i+1]-1; the first group_shared[i] tokens
    // of each of them sit in the same physical blocks (those of the group's
    // first sequence).  The prefix pass covers those tokens once per group.
    const int32_t* group_first;   // [num_groups + 1]
    const int32_t* group_shared;  // [num_groups]
    int num_groups;
    int max_group_size;           // prefix-pass grid covers groups up to this many sequences
    int max_shared;               // ... and shared runs up to this many tokens
    // Membership decided once per call by group_members_kernel (nullptr: no
    // groups): member[s] = (group index + 1, shared tokens) when sequence s
    // takes its group's prefix result, (0, 0) otherwise.
    const int2* member;
    // Nonzero: a decode kernel takes its (sequence, partition) unit from its
    // place in the grid in longest-first order (lpt_unit) instead of (z, y).
    int lpt;
    // Non-null: the kernel merges a row's split-K partials itself, in the CTA
    // that writes the row's last partial (split_arrive / merge_row_warp), and
    // no reduce kernel runs.  One word per (sequence, query head) row; stamp
    // identifies the call (48 bits).
    unsigned long long* split_count;
    unsigned long long stamp;
};

// A chunk of new tokens per sequence (causal): sequence s owns query rows
// query_start[s] .. query_start[s+1]-1, the last tokens of its context.
struct ChunkParams {
    const int32_t* query_start;  // [S + 1]
    int T;                       // query rows in q / out
    int max_query_len;           // host bound on query_start[s+1] - query_start[s]
    int nparts;                  // partitions of the longest context
};

// Which tokens one (sequence, partition) unit covers and where its result goes.
//   member  -- the sequence belongs to a valid shared-prefix group; its first
//              `shared` tokens are done by the prefix pass in npre partials
//              (slots 0..npre-1), its own partitions follow from slot npre.
//   direct  -- a lone partition of a non-member: write the output itself.
struct Unit {
    int L, shared, npre, nsuf, t_begin, t_end, slot;
    bool member, direct;
};

__device__ __forceinline__ int find_group(const AttnParams& p, int s) {
    if (p.num_groups <= 0) return -1;
    if (s < p.group_first[0] || s >= p.group_first[p.num_groups]) return -1;
    int lo = 0, hi = p.num_groups;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (p.group_first[mid] <= s) lo = mid;
        else hi = mid;
    }
    return lo;
}

// Shared length of group gi for a member whose context is L tokens, or -1 if
// the group's description is unusable for it (then it is treated as a
// non-member and the bad value recorded).
__device__ __forceinline__ int group_shared_len(const AttnParams& p, int gi, int L, bool report) {
    const int sh = p.group_shared[gi];
    if (sh < 0 || sh % p.bs != 0 || sh > L) {
        if (report) flag_error(4u /* PKV_DEVERR_CONTEXT */);
        return -1;
    }
    if (sh > p.max_shared) {
        if (report) flag_error(16u /* PKV_DEVERR_GROUP */);
        return -1;
    }
    return sh;
}


// Whether the first `shared / bs` block-table entries of sequence s are those
// of sequence `first` (the group's first sequence, whose table the prefix
// pass reads): only sequences that really hold the same blocks may share the
// prefix result (openeuler.csdn.net PagedAttention explainer 6.1;
// aiknowledge.cn "2.2 PagedAttention 与 KV Cache 分页管理" 2.2.8).
// Warp-collective: every lane calls it with the same s, first and shared
// (shared <= max_blocks_per_seq * bs, so both rows are read in bounds).
__device__ __forceinline__ bool same_leading_blocks(const int32_t* block_tables, int maxB, int bs, int s, int first,
                                                    int shared, int lane) {
    if (s == first) return true;
    const int n = shared / bs;
    const int32_t* a = block_tables + (int64_t)s * maxB;
    const int32_t* b = block_tables + (int64_t)first * maxB;
    bool same = true;
    for (int j = lane; j < n; j += 32) same = same && a[j] == b[j];
    return __all_sync(0xffffffffu, same);
}

// The group's first sequence as the prefix pass uses it (clamped into the batch).
__device__ __forceinline__ int group_first_seq(const int32_t* group_first, int gi, int S) {
    return max(0, min(group_first[gi], S));
}

// Context length of sequence s, clamped into [0, max_len]; an out-of-range
// value is recorded once per sequence (by the unit that owns partition 0).
__device__ __forceinline__ int load_context_len(const AttnParams& p, int s, bool report) {
    int L = p.context_lens[s];
    if (L < 0 || L > p.max_len) {
        if (report) flag_error(4u /* PKV_DEVERR_CONTEXT */);
        L = L < 0 ? 0 : p.max_len;
    }
    return L;
}

__device__ __forceinline__ Unit resolve_unit(const AttnParams& p, int s, int part, bool report) {
    Unit u;
    u.L = load_context_len(p, s, report);
    u.shared = 0;
    u.member = false;
    if (p.member != nullptr) {
        const int2 m = p.member[s];
        if (m.x > 0 && m.y > 0 && m.y <= u.L) {
            u.shared = m.y;
            u.member = true;
        }
    }
    u.npre = (u.shared + p.P - 1) / p.P;
    u.nsuf = (u.L - u.shared + p.P - 1) / p.P;
    u.t_begin = u.shared + part * p.P;
    u.t_end = min(u.L, u.t_begin + p.P);
    u.slot = u.npre + part;
    u.direct = !u.member && u.nsuf == 1;
    return u;
}

// Longest-first dispatch of a call's (sequence, partition) units.
//
// The hardware starts a grid's CTAs roughly in grid order, and a call's units
// run from 1 to P tokens (each sequence's last partition is the short one):
// a long unit started among the last CTAs sets the end of the kernel.  A
// decode kernel may instead take the unit of
// rank r, its place in the (y, z) plane of the grid (r = z * gridDim.y + y;
// every rank has gridDim.x CTAs, one per head group, started together).  A
// sequence's own tokens are its context less the prefix a shared-prefix
// group member takes from the prefix pass (AttnParams::member):
//   ranks 0 .. F-1      the full partitions (P own tokens), in sequence order;
//   ranks F .. F+R-1    the last partition of each sequence whose own length
//                       is not a multiple of P, and partition 0 of each empty
//                       sequence, longest first (lengths in kLptBins bins of
//                       about P/kLptBins tokens; ties in sequence order);
//   higher ranks        no unit (the grid has nparts * S ranks).
// These are exactly the units that partition order has (part < ceil(own/P),
// or part 0 of an empty sequence), so resolve_unit and the split-K reduce
// see the same (s, part) pairs.  One warp derives the order from
// context_lens (clamped like load_context_len) and the membership with
// shuffles and a radix select over the bins (lpt_unit, warp-collective);
// lpt_unit_cta hands the answer to the CTA's other warps.  The host sets p.lpt = PER, the sequences
// per lane (1, 2, 4 or 8: S <= 32 * PER), or 0 for grid order.
constexpr int kLptBins = 256;  // 8-bit bin index
constexpr int kLptPerLane = 8;  // largest PER

// floor(L / P) for 0 <= L < 2^24 from a float reciprocal of P (within one of
// the quotient there), corrected to the exact value.
__device__ __forceinline__ int lpt_div(int L, int P, float inv_p) {
    int q = __float2int_rz(__int2float_rn(L) * inv_p);
    const int r = L - q * P;
    q += r < 0 ? -1 : (r >= P ? 1 : 0);
    return q;
}

// The unit (s, part) of rank r over context_lens[0 .. S-1] (and member, if
// not null, as resolve_unit reads it), or (-1, -1); S <= 32 * PER.
template <int PER>
__device__ __noinline__ int2 lpt_unit(const int32_t* context_lens, const int2* member, int S, int P, int max_len,
                                      int r) {
    const int lane = threadIdx.x & 31;
    const int s0 = min(S, lane * PER), s1 = min(S, s0 + PER);  // this lane's sequences
    const bool small = max_len < (1 << 24);
    const float inv_p = __frcp_rn((float)P);
    int len[PER], own_len[PER], f[PER];  // clamped lengths (-1: no sequence); own tokens; full partitions
    int fsum = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        len[i] = -1;
        own_len[i] = 0;
        f[i] = 0;
        if (s0 + i < s1) {
            const int L = context_lens[s0 + i];
            len[i] = L < 0 ? 0 : (L > max_len ? max_len : L);
            own_len[i] = len[i];
            if (member != nullptr) {
                const int2 m = member[s0 + i];
                if (m.x > 0 && m.y > 0 && m.y <= len[i]) own_len[i] -= m.y;
            }
        }
    }
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        if (own_len[i] > 0) f[i] = small ? lpt_div(own_len[i], P, inv_p) : own_len[i] / P;
        fsum += f[i];
    }
    int x = fsum;  // inclusive prefix over lanes = over sequences
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
    }
    const int F = __shfl_sync(0xffffffffu, x, 31);
    int s = -1, part = -1;
    if (r < F) {
        const bool own = r >= x - fsum && r < x;
        if (own) {
            int acc = x - fsum;
#pragma unroll
            for (int i = 0; i < PER; ++i) {
                if (r >= acc && r < acc + f[i]) {
                    s = s0 + i;
                    part = r - acc;
                }
                acc += f[i];
            }
        }
        const int src = __ffs(__ballot_sync(0xffffffffu, own)) - 1;
        return make_int2(__shfl_sync(0xffffffffu, s, src), __shfl_sync(0xffffffffu, part, src));
    }
    // Bin of each sequence's short last partition (-1: none).
    int bin[PER];
    int psum = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int rem = own_len[i] - f[i] * P;
        bin[i] = len[i] < 0 || (rem == 0 && len[i] != 0) ? -1
                 : rem == 0                                ? 0
                                                           : min(kLptBins - 1, 1 + __float2int_rz(__int2float_rn(rem - 1) * inv_p *
                                                                                                  (kLptBins - 1)));
        psum += bin[i] >= 0 ? 1 : 0;
    }
    int k = r - F;
    if (k >= (int)__reduce_add_sync(0xffffffffu, (unsigned)psum)) return make_int2(-1, -1);
    // The bin of the k-th longest short unit, most significant bit first.
    int sel = 0;
#pragma unroll
    for (int bit = 7; bit >= 0; --bit) {
        const int want = (sel >> bit) | 1;
        int c = 0;
#pragma unroll
        for (int i = 0; i < PER; ++i) c += (bin[i] >> bit) == want ? 1 : 0;
        c = (int)__reduce_add_sync(0xffffffffu, (unsigned)c);
        if (k < c) sel |= 1 << bit;
        else k -= c;
    }
    // ... and the k-th sequence of that bin in sequence order.
    int m = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) m += bin[i] == sel ? 1 : 0;
    x = m;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
    }
    const bool own = k >= x - m && k < x;
    if (own) {
        int acc = x - m;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            if (bin[i] == sel) {
                if (acc == k) {
                    s = s0 + i;
                    part = f[i];
                }
                ++acc;
            }
        }
    }
    const int src = __ffs(__ballot_sync(0xffffffffu, own)) - 1;
    return make_int2(__shfl_sync(0xffffffffu, s, src), __shfl_sync(0xffffffffu, part, src));
}

// lpt_unit for rank r, computed by warp 0 and read by every warp of the CTA
// (block-collective: call before any warp leaves).  lpt = PER.
__device__ __forceinline__ int2 lpt_unit_cta(const AttnParams& p, int r) {
    __shared__ int2 pick;
    if (threadIdx.x < 32) {
        int2 u;
        switch (p.lpt) {
            case 1: u = lpt_unit<1>(p.context_lens, p.member, p.S, p.P, p.max_len, r); break;
            case 2: u = lpt_unit<2>(p.context_lens, p.member, p.S, p.P, p.max_len, r); break;
            case 4: u = lpt_unit<4>(p.context_lens, p.member, p.S, p.P, p.max_len, r); break;
            default: u = lpt_unit<kLptPerLane>(p.context_lens, p.member, p.S, p.P, p.max_len, r); break;
        }
        if (threadIdx.x == 0) pick = u;
    }
    __syncthreads();
    return pick;
}

// Split-K merge inside the decode kernel.
//
// Each of a row's n partials arrives at the row's counter word after writing
// its (o, m, l); the arrival that completes the count merges the row (the
// classic last-block pattern: a fence before the arrival, a fence and L1-
// bypassing loads after it; no thread waits for another).  A word holds the
// call's 48-bit stamp above a 16-bit count.  A word from another call (any
// other stamp, stale workspace contents included) counts as zero, so the
// workspace needs no initialisation; the completing arrival stores (stamp, 0),
// so a CUDA graph that replays one stamp starts every replay from zero.
// `seen` is the word as read before the partial was written (split_peek):
// usually still current, so one exchange settles the arrival.  Returns this
// arrival's count (1 .. n), 0 if the word could not be updated.
__device__ __forceinline__ unsigned long long split_peek(const unsigned long long* word) { return __ldcg(word); }

__device__ __forceinline__ int split_arrive(unsigned long long* word, unsigned long long stamp, int n,
                                            unsigned long long seen) {
    unsigned long long old = seen;
    // Each failed exchange after the first is another arrival of this row's n
    // succeeding (the first may also fail on a stale `seen`).
    for (int it = 0; it <= n + 1; ++it) {
        const int cnt = (old >> 16) == stamp ? (int)(old & 0xffffu) + 1 : 1;
        const unsigned long long want = (stamp << 16) | (unsigned long long)(cnt >= n ? 0 : cnt);
        const unsigned long long got = atomicCAS(word, old, want);
        if (got == old) return cnt;
        old = got;
    }
    return 0;
}

// One warp merges the n <= 32 partials of a row (slots base .. base+n-1 of
// ws_o / ws_ml) into dst: the arithmetic and order of splitk_reduce_warp_kernel
// (weights 2^(m_i - M) from a warp maximum, a butterfly sum for the
// denominator, the weighted outputs summed in slot order).
template <typename T, int D>
__device__ __forceinline__ void merge_row_warp(const float* ws_o, const float* ws_ml, int64_t base, int n, T* dst,
                                               int lane) {
    constexpr int KPL = D / 32;  // 2 or 4 floats per lane
    const float2 mlv = lane < n ? __ldcg(reinterpret_cast<const float2*>(ws_ml + (base + lane) * 2))
                                : make_float2(-INFINITY, 0.f);
    float M = mlv.x;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    const float w_lane = lane < n ? ex2(mlv.x - M) : 0.f;
    float den = w_lane * (lane < n ? mlv.y : 0.f);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
    float acc[KPL];
#pragma unroll
    for (int k = 0; k < KPL; ++k) acc[k] = 0.f;
    const float* o = ws_o + base * D + lane * KPL;
    for (int i = 0; i < n; ++i) {
        const float w = __shfl_sync(0xffffffffu, w_lane, i);
        float x[KPL];
        if constexpr (KPL == 4) {
            const float4 y = __ldcg(reinterpret_cast<const float4*>(o + (int64_t)i * D));
            x[0] = y.x; x[1] = y.y; x[2] = y.z; x[3] = y.w;
        } else {
            const float2 y = __ldcg(reinterpret_cast<const float2*>(o + (int64_t)i * D));
            x[0] = y.x; x[1] = y.y;
        }
#pragma unroll
        for (int k = 0; k < KPL; ++k) acc[k] += w * x[k];
    }
    const float inv = 1.f / den;
#pragma unroll
    for (int k = 0; k < KPL; ++k) dst[lane * KPL + k] = static_cast<T>(acc[k] * inv);
}

// After a warp wrote partial slot u.slot of `row`: arrive, and merge the row
// if this was its last partial (warp-collective).  seen: split_peek of the
// row's word by lane 0 before the partial was written.
template <typename T, int D>
__device__ __forceinline__ void merge_if_last(const AttnParams& p, int64_t row, int n, int lane,
                                              unsigned long long seen) {
    __threadfence();
    __syncwarp();
    int cnt = 0;
    if (lane == 0) {
        cnt = split_arrive(p.split_count + row, p.stamp, n, seen);
        if (cnt == 0) flag_error(32u /* PKV_DEVERR_SPLIT */);
    }
    cnt = __shfl_sync(0xffffffffu, cnt, 0);
    if (cnt != n) return;
    __threadfence();
    merge_row_warp<T, D>(p.ws_o, p.ws_ml, row * p.maxP, n, reinterpret_cast<T*>(p.out) + row * D, lane);
}

// Shared-prefix membership of every sequence of a call, decided once before
// the attention kernels run (one warp per sequence, 8 per CTA), so that the
// decode kernels, the prefix pass and the reduce all read the same answer
// from member[s] (see AttnParams::member).  A sequence of group gi takes the
// prefix result when the group's shared length is usable for it (a multiple
// of block_size within its context and within max_shared_len), it lies
// within max_group_size of the group's first sequence (the prefix pass's
// grid), and its first shared/block_size table entries are the first
// sequence's -- the blocks the prefix pass reads.  Failures are recorded once
// per sequence; such a sequence attends to its whole context through its own
// table.
__global__ void __launch_bounds__(256) group_members_kernel(const AttnParams p, int2* member) {
    const int lane = threadIdx.x & 31;
    const int s = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (s >= p.S) return;
    int2 m = make_int2(0, 0);
    const int L = load_context_len(p, s, false);  // a bad length is reported by the decode kernels
    const int gi = find_group(p, s);
    if (gi >= 0) {
        const int sh = group_shared_len(p, gi, L, lane == 0);
        if (sh > 0) {
            const int first = group_first_seq(p.group_first, gi, p.S);
            const bool within = s - first < p.max_group_size;
            const bool same = same_leading_blocks(p.block_tables, p.maxB, p.bs, s, first, sh, lane);
            if (within && same) m = make_int2(gi + 1, sh);
            else if (lane == 0) flag_error(16u /* PKV_DEVERR_GROUP */);
        }
    }
    if (lane == 0) member[s] = m;
}

// Block-table window held in registers: lane l holds entry (first + base + l)
// of the sequence's table, for the blocks one work unit touches.  All lanes
// call get() with the same (warp-uniform) logical index, in non-decreasing
// order.
struct BlockWindow {
    const int32_t* row;  // this sequence's table row, offset to the unit's first block
    int count;           // blocks of the unit
    int base;            // index of the entry lane 0 holds
    int mine;

    __device__ __forceinline__ void init(const int32_t* table_row, int first, int n, int lane) {
        row = table_row + first;
        count = n;
        base = 0;
        mine = lane < n ? row[lane] : 0;
    }
    __device__ __forceinline__ int get(int j, int lane, int num_blocks) {
        if (j >= base + 32) {
            base = j;
            mine = base + lane < count ? row[base + lane] : 0;
        }
        int b = __shfl_sync(0xffffffffu, mine, j - base);
        if ((unsigned)b >= (unsigned)num_blocks) {
            if (lane == 0) flag_error(1u /* PKV_DEVERR_BLOCK_ID */);
            b = 0;  // read a valid block instead; the output is flagged meaningless
        }
        return b;
    }
};

}  // namespace pkv
