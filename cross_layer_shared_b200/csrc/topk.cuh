// Launch interface of the top-k kernels (internal to libsa).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "status.cuh"

namespace sa {

size_t topk_rows_smem_bytes();

// One CTA per row: exact top-k with ties to the lower index, ascending output.
cudaError_t launch_topk_rows(const float* scores, int64_t ld, const int32_t* n_valid, int Nq, int n_max, int k,
                             int32_t* idx, float* top_scores, DeviceStatus* status, cudaStream_t stream);

// Few long rows (Nq <= num_sms / 2, n_max > 8192): one cluster of CTAs per row.
bool topk_use_split(int Nq, int n_max, int num_sms);
size_t topk_split_ws_bytes(int Nq, int n_max, int num_sms);
cudaError_t launch_topk_split(const float* scores, int64_t ld, const int32_t* n_valid, int Nq, int n_max, int k,
                              int32_t* idx, float* top_scores, DeviceStatus* status, void* scratch, int num_sms,
                              cudaStream_t stream);

// Dynamic k by routing mass (topk_dynamic.cu), one CTA per row, over the
// row's top k_max (sel_idx ascending then -1, sel_s their scores) from the
// kernels above: idx [Nq, k_max] keeps the m entries reaching tau of the
// row's total score in the top-k order, then -1; counts [Nq] = m.
// k_max <= 4096.
size_t topk_dynamic_smem_bytes(int k_max);
cudaError_t launch_topk_dynamic(const float* scores, int64_t ld, const int32_t* n_valid, int Nq, int n_max,
                                const int32_t* sel_idx, const float* sel_s, int k_max, double tau, int32_t* idx,
                                int32_t* counts, DeviceStatus* status, cudaStream_t stream);

}  // namespace sa
