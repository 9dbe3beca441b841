// Device fault word of libpkv (PKV_FAULT_* bits of pkv.h).  Every kernel of the library is
// compiled into the one translation unit pkv_cuda.cu, which includes this header once.
#pragma once

namespace pkv {
__device__ unsigned int g_faults = 0;

// The bits, as pkv.h numbers them.
constexpr unsigned kFaultBadLen = 0x1u;     // context length outside [1, maxB*16]
constexpr unsigned kFaultBadBlock = 0x2u;   // block-table entry outside the pool
constexpr unsigned kFaultBadSlot = 0x4u;    // slot outside the pool (or not position L-1's)
constexpr unsigned kFaultBadPair = 0x8u;    // copy / swap pair naming a block outside a pool
constexpr unsigned kFaultTimeout = 0x10u;   // a bounded shared-memory barrier wait gave up
constexpr unsigned kFaultDuplicate = 0x20u; // a repeated slot or copy destination, or a copy
                                            // destination that is also a source
constexpr unsigned kFaultBadScale = 0x40u;  // an FP8 scale that is not finite and > 0
}  // namespace pkv
