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
