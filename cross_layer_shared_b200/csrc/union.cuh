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

namespace sa {

// Priority list per query block of q_block queries (CoSA's proxy under the
// hit-count reading): order[i, 0:nT] = the table kv_indices[kv_indptr[0] :
// kv_indptr[1]] ordered by hit count, larger first, ties by ascending id.
// Shared memory: kap_order_smem(ceil(S/block)) bytes per CTA.
constexpr int kKapMaxBlocks = 16384;
size_t kap_order_smem(int nb);
cudaError_t launch_kap_order(const int32_t* idx, int Nq, int k, int S, int block, int q_block,
                             const int32_t* kv_indptr, const int32_t* kv_indices, int32_t* order, int64_t ld,
                             DeviceStatus* status, cudaStream_t stream);

}  // namespace sa
