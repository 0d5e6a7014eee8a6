// Launch interface of the block-union kernels (internal to libsa).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "status.cuh"

namespace sa {

// mark: ceil(S/block) bytes of scratch.
cudaError_t launch_block_union(const int32_t* idx, int Nq, int k, int S, int block, int Hkv, uint8_t* mark,
                               int32_t* kv_indptr, int32_t* kv_indices, DeviceStatus* status,
                               cudaStream_t stream);

}  // namespace sa
