// kv_append: write each new token's K and V (all kv heads) into its slot.
// openeuler.csdn.net PagedAttention explainer 2.2 (one new K/V cached per
// step); aiknowledge.cn "2.2 PagedAttention 与 KV Cache 分页管理" 2.2.3 (the
// token goes to its sequence's last block at offset t % block_size).
//
// One thread moves one 16-byte vector of K and the matching one of V; a warp
// covers 512 contiguous bytes of a (token, head) row, so loads and stores are
// fully coalesced.  Pure byte copy: bit-exact.
#pragma once
#include "common.cuh"

namespace pkv {

struct AppendParams {
    const uint4* k_new;   // [T][Hkv][D] as 16-byte vectors
    const uint4* v_new;
    uint4* k_pool;        // [NB][Hkv][bs][D]
    uint4* v_pool;
    const int64_t* slot_mapping;
    int64_t total_vecs;   // T * Hkv * vecs_per_row
    int vecs_per_row;     // D * elem_size / 16
    int Hkv;
    int bs;
    int64_t num_slots;    // NB * bs
};

__global__ void __launch_bounds__(256) kv_append_kernel(const AppendParams p) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < p.total_vecs; i += stride) {
        const int64_t row = i / p.vecs_per_row;          // (token, head)
        const int vec = (int)(i - row * p.vecs_per_row);
        const int64_t tok = row / p.Hkv;
        const int head = (int)(row - tok * p.Hkv);
        const int64_t slot = p.slot_mapping[tok];
        if (slot < 0) continue;
        if (slot >= p.num_slots) {
            flag_error(2u /* PKV_DEVERR_SLOT */);
            continue;
        }
        const int64_t blk = slot / p.bs;
        const int64_t off = slot - blk * p.bs;
        const int64_t dst = ((blk * p.Hkv + head) * p.bs + off) * p.vecs_per_row + vec;
        p.k_pool[dst] = p.k_new[i];
        p.v_pool[dst] = p.v_new[i];
    }
}

// Quantizing append into FP8 E4M3 pools: code = e4m3(x * inv_scale) computed
// in fp32, round to nearest even, saturated to +-448.  One thread per 16
// elements of a (token, head) row (16 bytes of codes).
struct AppendFp8Params {
    const void* k_new;   // [T][Hkv][D] of S
    const void* v_new;
    uint4* k_pool;       // [NB][Hkv][bs][D] codes
    uint4* v_pool;
    const int64_t* slot_mapping;
    int64_t total_vecs;  // T * Hkv * (D / 16)
    int vecs_per_row;    // D / 16
    int Hkv;
    int bs;
    int64_t num_slots;
    float k_inv, v_inv;
};

template <typename S>
__device__ __forceinline__ uint4 quantize16(const S* src, float inv) {
    float f[16];
    load_slice<S, 16>(src, f);
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t lo = f32x2_to_e4m3x2(f[4 * i] * inv, f[4 * i + 1] * inv);
        const uint32_t hi = f32x2_to_e4m3x2(f[4 * i + 2] * inv, f[4 * i + 3] * inv);
        w[i] = lo | (hi << 16);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

template <typename S>
__global__ void __launch_bounds__(256) kv_append_fp8_kernel(const AppendFp8Params p) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < p.total_vecs; i += stride) {
        const int64_t row = i / p.vecs_per_row;
        const int vec = (int)(i - row * p.vecs_per_row);
        const int64_t tok = row / p.Hkv;
        const int head = (int)(row - tok * p.Hkv);
        const int64_t slot = p.slot_mapping[tok];
        if (slot < 0) continue;
        if (slot >= p.num_slots) {
            flag_error(2u /* PKV_DEVERR_SLOT */);
            continue;
        }
        const int64_t blk = slot / p.bs;
        const int64_t off = slot - blk * p.bs;
        const int64_t dst = ((blk * p.Hkv + head) * p.bs + off) * p.vecs_per_row + vec;
        p.k_pool[dst] = quantize16(reinterpret_cast<const S*>(p.k_new) + i * 16, p.k_inv);
        p.v_pool[dst] = quantize16(reinterpret_cast<const S*>(p.v_new) + i * 16, p.v_inv);
    }
}

}  // namespace pkv
