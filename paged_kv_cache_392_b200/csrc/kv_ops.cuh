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
// Both are plain bandwidth work: 16-byte vector loads and stores, coalesced along the head
// dimension; every index is range-checked before it is used.  Both also check the call's
// distinctness rules on the device and skip what breaks them, whatever the order in which
// the CTAs run: a slot given to two tokens (both are skipped), a copy destination named by
// two pairs (both skipped) or a destination that is also a source (that pair skipped).  The
// skipped entries set PKV_FAULT_DUPLICATE; the others are written as usual.
#pragma once
#include <cstdint>

#include "faults.cuh"

namespace pkv {

constexpr int kWriteThreads = 256;   // threads per kv_write CTA (8 warps)
constexpr int kTileTokens = 32;      // tokens per kv_write tile: lane i <-> token i of the tile
constexpr int kSlotChunk = 2048;     // slots staged in shared memory per pass of the check

struct TileSlots {
    int64_t chunk[kSlotChunk];
    int64_t slot[kTileTokens];       // the tile's slots (-1 past the end of the call)
    int count[kWriteThreads];
    unsigned dup_mask;               // bit i: token i of the tile shares its slot
};

// Slots of tokens t0 .. t0+31 of a call, and which of them another token of the call also
// names: the whole slot_mapping streams through shared memory in chunks, each warp counts
// the matches of lane i's slot in its share of a chunk, and a token whose slot (not -1)
// appears more than once is a duplicate.  Called by all kWriteThreads threads of the CTA.
// Cost: T comparisons per tile token, so T * T over the call.
__device__ __forceinline__ void tile_duplicate_slots(const int64_t *slot_mapping, int64_t T,
                                                     int64_t t0, TileSlots &ts) {
    constexpr int kWarps = kWriteThreads / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t mine = t0 + lane < T ? slot_mapping[t0 + lane] : -1;
    int cnt = 0;
    for (int64_t c0 = 0; c0 < T; c0 += kSlotChunk) {
        const int n = (int)(T - c0 < kSlotChunk ? T - c0 : kSlotChunk);
        __syncthreads();  // the previous chunk is no longer read
        for (int j = threadIdx.x; j < n; j += kWriteThreads) ts.chunk[j] = slot_mapping[c0 + j];
        __syncthreads();
        for (int j = warp; j < n; j += kWarps) cnt += ts.chunk[j] == mine;
    }
    ts.count[threadIdx.x] = cnt;
    __syncthreads();
    if (warp == 0) {
        int total = 0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) total += ts.count[w * 32 + lane];
        ts.slot[lane] = mine;
        const unsigned m = __ballot_sync(0xffffffffu, mine != -1 && total > 1);
        if (lane == 0) ts.dup_mask = m;
    }
    __syncthreads();
}

struct KvWriteParams {
    const uint4 *k_new;  // [T][H_kv][D] as 16-byte vectors
    const uint4 *v_new;
    const int64_t *slot_mapping;
    uint4 *k_pool;       // [NB][H_kv][B][D]
    uint4 *v_pool;
    int32_t T, Hkv, NB;
    int32_t vpr;         // 16-byte vectors per row (D * elem_size / 16)
    int32_t bshift;      // log2 B: tokens per block (16 or 32)
};

// grid.x = tile of kTileTokens tokens, grid.y = slice of the tile's vectors.  Within a tile
// the vectors run (pool, token, head, 16-byte column), so a warp's stores are coalesced.
__global__ void __launch_bounds__(kWriteThreads) kv_write_kernel(const KvWriteParams p) {
    __shared__ TileSlots ts;
    const int64_t t0 = (int64_t)blockIdx.x * kTileTokens;
    tile_duplicate_slots(p.slot_mapping, p.T, t0, ts);
    const int ntok = (int)(p.T - t0 < kTileTokens ? p.T - t0 : kTileTokens);
    const int per_tok = p.Hkv * p.vpr;         // vectors of one token in one pool
    const int half = ntok * per_tok;
    const int per_cta = (2 * half + gridDim.y - 1) / gridDim.y;
    const int end = min(2 * half, (int)(blockIdx.y + 1) * per_cta);
    for (int i = blockIdx.y * per_cta + threadIdx.x; i < end; i += kWriteThreads) {
        const int which = i >= half;
        const int r = which ? i - half : i;
        const int tl = r / per_tok, hc = r % per_tok;
        const int64_t slot = ts.slot[tl];
        if (slot == -1) continue;
        const bool reporter = which == 0 && hc == 0;   // one report per token
        if (slot < 0 || slot >= ((int64_t)p.NB << p.bshift)) {
            if (reporter) atomicOr(&g_faults, kFaultBadSlot);
            continue;
        }
        if ((ts.dup_mask >> tl) & 1u) {
            if (reporter) atomicOr(&g_faults, kFaultDuplicate);
            continue;
        }
        const int h = hc / p.vpr, c = hc % p.vpr;
        const int64_t dst = ((((slot >> p.bshift) * p.Hkv + h) << p.bshift) +
                             (slot & ((1 << p.bshift) - 1))) * p.vpr + c;
        const int64_t src = (t0 + tl) * per_tok + hc;
        if (which == 0)
            p.k_pool[dst] = p.k_new[src];
        else
            p.v_pool[dst] = p.v_new[src];
    }
}

// Whether pair i's destination is also the destination of another pair, or (when sources
// and destinations live in the same pool) the source of any pair, itself included.  Pairs
// are int32 [P][2] (source, destination).  Called by all threads of the CTA.
__device__ __forceinline__ bool pair_conflicts(const int32_t *pairs, int P, int i, int32_t dst,
                                               bool same_pool) {
    bool c = false;
    for (int j = threadIdx.x; j < P; j += blockDim.x) {
        const int32_t sj = pairs[2 * j], dj = pairs[2 * j + 1];
        c |= (dj == dst && j != i) || (same_pool && sj == dst);
    }
    return __syncthreads_or(c) != 0;
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
    const bool reporter = threadIdx.x == 0 && blockIdx.y == 0 && pool == 0;
    const int32_t src = p.pairs[2 * pair];
    const int32_t dst = p.pairs[2 * pair + 1];
    if ((unsigned)src >= (unsigned)p.NB || (unsigned)dst >= (unsigned)p.NB) {
        if (reporter) atomicOr(&g_faults, kFaultBadPair);
        return;
    }
    if (pair_conflicts(p.pairs, p.P, pair, dst, true)) {
        if (reporter) atomicOr(&g_faults, kFaultDuplicate);
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
    const bool reporter = threadIdx.x == 0 && blockIdx.y == 0 && pool == 0;
    if ((unsigned)src >= (unsigned)p.nb_src || (unsigned)dst >= (unsigned)p.nb_dst) {
        if (reporter) atomicOr(&g_faults, kFaultBadPair);
        return;
    }
    if (pair_conflicts(p.pairs, p.P, pair, dst, false)) {
        if (reporter) atomicOr(&g_faults, kFaultDuplicate);
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
