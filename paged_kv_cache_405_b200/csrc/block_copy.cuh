// block_copy: copy-on-write support -- duplicate whole physical blocks.
// openeuler.csdn.net PagedAttention explainer 6.2: a write into a block other
// sequences still use first copies that one block; the original stays as it
// is for them.  agent.csdn.net PagedAttention blog 2.2: forked samples/beams.
//
// Grid: x = pair, y = slices of the block.  Each thread moves 16-byte vectors
// of K and V; a (src, dst) block is contiguous (all kv heads x block_size x
// head_dim), so every warp access is 512 contiguous bytes.  Bit-exact.
#pragma once
#include "common.cuh"

namespace pkv {

struct CopyParams {
    uint4* k_pool;
    uint4* v_pool;
    const int32_t* pairs;   // [n][2] (src, dst)
    int64_t block_vecs;     // Hkv * bs * D * elem_size / 16
    int num_blocks;
};

__global__ void __launch_bounds__(256) block_copy_kernel(const CopyParams p) {
    const int pair = blockIdx.x;
    const int src = p.pairs[2 * pair];
    const int dst = p.pairs[2 * pair + 1];
    if (src < 0 || src >= p.num_blocks || dst < 0 || dst >= p.num_blocks) {
        if (threadIdx.x == 0 && blockIdx.y == 0) flag_error(1u /* PKV_DEVERR_BLOCK_ID */);
        return;
    }
    const uint4* ks = p.k_pool + (int64_t)src * p.block_vecs;
    const uint4* vs = p.v_pool + (int64_t)src * p.block_vecs;
    uint4* kd = p.k_pool + (int64_t)dst * p.block_vecs;
    uint4* vd = p.v_pool + (int64_t)dst * p.block_vecs;
    const int64_t stride = (int64_t)gridDim.y * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.y * blockDim.x + threadIdx.x; i < p.block_vecs; i += stride) {
        uint4 a = ks[i];
        uint4 b = vs[i];
        kd[i] = a;
        vd[i] = b;
    }
}

}  // namespace pkv
