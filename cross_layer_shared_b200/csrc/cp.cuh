// Launch interface of the context-parallel decode kernels (internal to libsa).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "status.cuh"

namespace sa {

// Per-sequence state of the radix exchange (in the workspace): the key
// prefix found so far, the number of keys still needed within it, and
// whether all ranks together hold no more than k valid keys.
struct CpRadixState {
  uint32_t prefix;
  int need;
  int all;
  int pad;
};
// Level 0, 1, 2 of the exchange: the previous level's threshold from the
// gathered histograms (levels 1, 2), then this rank's histogram of the
// level's digit into hist_out [B][4096] (levels 0, 1) or [B][256] (level 2).
cudaError_t launch_cp_radix_level(const float* scores, int64_t ld, const int32_t* n_local, int B, int k, int N,
                                  int level, const int32_t* gathered, int64_t rank_stride, CpRadixState* state,
                                  int32_t* hist_out, DeviceStatus* status, cudaStream_t stream);
// The last threshold, then this rank's share of the global top-k as local
// indices (ascending, -1 padded) and their count.
cudaError_t launch_cp_radix_finish(const float* scores, int64_t ld, const int32_t* n_local, int B, int k, int N,
                                   int rank, const int32_t* gathered, int64_t rank_stride, const CpRadixState* state,
                                   int32_t* local_idx, int32_t* count, DeviceStatus* status, cudaStream_t stream);

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
