// Read-bandwidth probe: the decode's memory pattern with the decode taken out.  Warps stream
// chunks of a device buffer into shared-memory rings with 1-D bulk copies and discard them,
// so its rate is what this GPU's memory system delivers to copies of that size scattered
// over the buffer: a read-only ceiling to set beside the copy-based peak.
#pragma once
#include <cstdint>

#include "attn_decode.cuh"

namespace pkv {

constexpr int kProbeWarps = 2;     // warps per CTA
constexpr int kProbeStages = 4;    // copies in flight per warp
// MurmurHash3's 32-bit finaliser (Appleby): a bijection on 32-bit integers that mixes every
// input bit into every output bit.
__device__ __forceinline__ uint32_t fmix32(uint32_t x) {
    x ^= x >> 16;
    x *= 0x85EBCA6Bu;
    x ^= x >> 13;
    x *= 0xC2B2AE35u;
    x ^= x >> 16;
    return x;
}

// Chunk k of the stream is chunk probe_scatter(k) of the buffer: a pseudo-random permutation
// of [0, n), n = 2^b, so that the copies in flight at any time are spread over the buffer the
// way the decode's shuffled blocks are.  A 4-round Feistel network on 2h bits (h = ceil(b/2);
// round function fmix32 of the right half and a round constant) is a permutation of
// [0, 2^2h), 2^2h being n or 2n; applying it again until the value is below n (cycle walking)
// keeps it a permutation of [0, n), after two steps on average.  (Simpler orders, such as an
// odd multiply with xor-shifts, left consecutive copies correlated enough to halve the rate
// with many 2 KiB copies in flight.)
__device__ __forceinline__ uint32_t probe_scatter(uint32_t k, uint32_t n, int h) {
    const uint32_t m = (1u << h) - 1u;
    uint32_t x = k;
    do {
        uint32_t l = x >> h, r = x & m;
#pragma unroll
        for (int i = 1; i <= 4; ++i) {
            const uint32_t t = l ^ (fmix32(r ^ (0x9E3779B9u * (uint32_t)i)) & m);
            l = r;
            r = t;
        }
        x = (l << h) | r;
    } while (x >= n);
    return x;
}

__global__ void __launch_bounds__(kProbeWarps * 32)
read_probe_kernel(const char *buf, uint32_t n, uint32_t chunk) {
    extern __shared__ __align__(16) unsigned char probe_ring[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    unsigned char *ring = probe_ring + (size_t)warp * kProbeStages * chunk;
    uint64_t *bars = reinterpret_cast<uint64_t *>(probe_ring +
                                                  (size_t)kProbeWarps * kProbeStages * chunk) +
                     warp * kProbeStages;
    const uint32_t gw = blockIdx.x * kProbeWarps + warp, nw = gridDim.x * kProbeWarps;
    if (lane == 0) {
#pragma unroll
        for (int i = 0; i < kProbeStages; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
    }
    __syncwarp();
    const uint64_t policy = l2_evict_first_policy();
    const int half = (__ffs(n) - 1 + 1) >> 1;   // ceil(b / 2) for n = 2^b
    const uint32_t mine = gw < n ? (n - gw + nw - 1) / nw : 0;   // this warp's chunks
    auto issue = [&](uint32_t i) {
        if (lane == 0) {
            const uint32_t c = probe_scatter(gw + i * nw, n, half);
            uint64_t *bar = &bars[i % kProbeStages];
            mbar_arrive_expect_tx(bar, chunk);
            bulk_g2s(ring + (i % kProbeStages) * chunk, buf + (size_t)c * chunk, chunk, bar,
                     policy);
        }
    };
    uint32_t issued = 0;
    for (; issued < (uint32_t)kProbeStages && issued < mine; ++issued) issue(issued);
    for (uint32_t i = 0; i < mine; ++i) {
        if (!mbar_wait_bounded(&bars[i % kProbeStages], (i / kProbeStages) & 1u,
                               kWaitTimeoutNs)) {
            if (lane == 0) atomicOr(&g_faults, kFaultTimeout);
            for (uint32_t b = i + 1; b < issued; ++b)
                (void)mbar_wait_bounded(&bars[b % kProbeStages], (b / kProbeStages) & 1u,
                                        kWaitTimeoutNs);
            return;
        }
        __syncwarp();
        if (issued < mine) {
            issue(issued);
            ++issued;
        }
    }
}

}  // namespace pkv
