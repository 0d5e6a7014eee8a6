// Launch interface of the context-parallel decode kernels (internal to libsa).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace sa {

// rank r's [B][k] candidates at cand_* + r*stride -> rows [B][N*k] (-inf
// where cand_idx < 0), n_valid[b] = N*k
cudaError_t launch_cp_gather(const float* cand_scores, const int32_t* cand_idx, int64_t stride, int N, int B, int k,
                             float* rows, int32_t* n_valid, cudaStream_t stream);
// sel [B][k] positions in a row (ascending, -1 padded) -> this rank's local
// indices [B][k] (ascending, -1 padded) and, if count is set, their number
cudaError_t launch_cp_local(const int32_t* sel, const int32_t* cand_idx, int64_t stride, int B, int k, int rank,
                            int32_t* local_idx, int32_t* count, cudaStream_t stream);
// part p: [rows][128] fp32 at parts + p*o_stride, [rows] (m, l) at ml +
// p*ml_stride -> O [rows][128] (fp32 or bf16)
cudaError_t launch_combine_partials(const float* parts, int64_t o_stride, const float2* ml, int64_t ml_stride, int P,
                                    int64_t rows, void* O, bool out_f32, cudaStream_t stream);

}  // namespace sa
