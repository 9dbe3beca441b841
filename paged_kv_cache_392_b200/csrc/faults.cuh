// Device fault word of libpkv (PKV_FAULT_* bits of pkv.h).  Every kernel of the library is
// compiled into the one translation unit pkv_cuda.cu, which includes this header once.
#pragma once

namespace pkv {
__device__ unsigned int g_faults = 0;
}  // namespace pkv
