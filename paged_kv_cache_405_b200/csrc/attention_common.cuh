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
    float scale_log2;          // softmax scale * log2(e)
};

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
