// KV-cache write and copy-on-write block copy kernels for sm_100a.
//
// kv_write ("Memory Optimization in LLM Serving with PagedAttention", section "How
// PagedAttention Works": blocks are filled on demand as generation proceeds): each new
// token's K and V rows go to the slot the block manager gave it; bytes are moved unchanged.
//
// kv_copy_blocks (same page, section "Advanced Capabilities: Memory Sharing with
// Copy-on-Write": a shared block is copied to a fresh block before a sequence writes into
// it): every (kv head, slot) of block src is copied to block dst, in both pools.
//
// Both are plain bandwidth work: 16-byte vector loads and stores, one thread per vector,
// coalesced along the head dimension; every index is range-checked before it is used.
#pragma once
#include <cstdint>

#include "faults.cuh"

namespace pkv {


struct KvWriteParams {
    const uint4 *k_new;  // [T][H_kv][D] as 16-byte vectors
    const uint4 *v_new;
    const int64_t *slot_mapping;
    uint4 *k_pool;       // [NB][H_kv][16][D]
    uint4 *v_pool;
    int32_t T, Hkv, NB;
    int32_t vpr;         // 16-byte vectors per row (D * elem_size / 16)
};

// One thread per 16-byte vector of K or V: index = ((which * T + t) * Hkv + h) * vpr + c.
__global__ void __launch_bounds__(256) kv_write_kernel(const KvWriteParams p) {
    const int64_t per = (int64_t)p.T * p.Hkv * p.vpr;
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= 2 * per) return;
    const int which = idx >= per;
    const int64_t rem = which ? idx - per : idx;
    const int c = (int)(rem % p.vpr);
    const int64_t th = rem / p.vpr;          // t * Hkv + h
    const int h = (int)(th % p.Hkv);
    const int64_t t = th / p.Hkv;
    const int64_t slot = p.slot_mapping[t];
    if (slot == -1) return;
    if (slot < 0 || slot >= (int64_t)p.NB * 16) {
        if (h == 0 && c == 0 && which == 0) atomicOr(&g_faults, 0x4u);
        return;
    }
    const int64_t blk = slot >> 4, off = slot & 15;
    const int64_t dst = ((blk * p.Hkv + h) * 16 + off) * p.vpr + c;
    if (which == 0)
        p.k_pool[dst] = p.k_new[rem];
    else
        p.v_pool[dst] = p.v_new[rem];
}

struct KvCopyParams {
    const int32_t *pairs;  // [P][2] (src, dst)
    uint4 *k_pool;
    uint4 *v_pool;
    int32_t P, NB;
    int64_t vpb;           // 16-byte vectors per block (H_kv * 16 * D * elem_size / 16)
};

constexpr int kCopyUnroll = 4;

// grid.x = pair * 2 + pool, grid.y = slice of kCopyUnroll * 256 vectors of the block.
__global__ void __launch_bounds__(256) kv_copy_blocks_kernel(const KvCopyParams p) {
    const int pair = blockIdx.x >> 1;
    const int pool = blockIdx.x & 1;
    const int32_t src = p.pairs[2 * pair];
    const int32_t dst = p.pairs[2 * pair + 1];
    if ((unsigned)src >= (unsigned)p.NB || (unsigned)dst >= (unsigned)p.NB) {
        if (threadIdx.x == 0 && blockIdx.y == 0 && pool == 0) atomicOr(&g_faults, 0x8u);
        return;
    }
    uint4 *base = pool ? p.v_pool : p.k_pool;
    const uint4 *s = base + (int64_t)src * p.vpb;
    uint4 *d = base + (int64_t)dst * p.vpb;
    const int64_t i0 = (int64_t)blockIdx.y * (kCopyUnroll * 256) + threadIdx.x;
    uint4 buf[kCopyUnroll];
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
        const int64_t i = i0 + u * 256;
        if (i < p.vpb) buf[u] = s[i];
    }
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
        const int64_t i = i0 + u * 256;
        if (i < p.vpb) d[i] = buf[u];
    }
}

// Swap of whole blocks between the device pools and a host pool (pinned, mapped memory
// reached over PCIe): "vLLM and PagedAttention: How Ideas from Operating Systems Accelerated
// LLM Inference" -- when memory runs short, whole sequences are evicted to CPU memory and
// brought back later.  For pair i, block dst of the destination pool becomes a byte copy of
// block src of the source pool, for K and for V.  One direction per launch.
struct KvSwapParams {
    const int32_t *pairs;  // [P][2] (src block, dst block)
    const uint4 *src_k;
    const uint4 *src_v;
    uint4 *dst_k;
    uint4 *dst_v;
    int32_t P, nb_src, nb_dst;
    int64_t vpb;           // 16-byte vectors per block
};

__global__ void __launch_bounds__(256) kv_swap_kernel(const KvSwapParams p) {
    const int pair = blockIdx.x >> 1;
    const int pool = blockIdx.x & 1;
    const int32_t src = p.pairs[2 * pair];
    const int32_t dst = p.pairs[2 * pair + 1];
    if ((unsigned)src >= (unsigned)p.nb_src || (unsigned)dst >= (unsigned)p.nb_dst) {
        if (threadIdx.x == 0 && blockIdx.y == 0 && pool == 0) atomicOr(&g_faults, 0x8u);
        return;
    }
    const uint4 *s = (pool ? p.src_v : p.src_k) + (int64_t)src * p.vpb;
    uint4 *d = (pool ? p.dst_v : p.dst_k) + (int64_t)dst * p.vpb;
    const int64_t i0 = (int64_t)blockIdx.y * (kCopyUnroll * 256) + threadIdx.x;
    uint4 buf[kCopyUnroll];
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
        const int64_t i = i0 + u * 256;
        if (i < p.vpb) buf[u] = s[i];
    }
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
        const int64_t i = i0 + u * 256;
        if (i < p.vpb) d[i] = buf[u];
    }
}

}  // namespace pkv
