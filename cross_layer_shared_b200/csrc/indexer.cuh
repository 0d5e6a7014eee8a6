// Launch interface of the indexer kernels (internal to libsa).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "status.cuh"

namespace sa {

struct IndexerArgs {
  const float* w;
  const int64_t* seq_off;
  const int32_t* seq_len;
  int B;
  int64_t n_tokens;
  int S_max;
  int H_I;
  int d_I;
  float* scores;
  int64_t ld;
  DeviceStatus* status;
};

// tm_ki: KI [n_tokens, d_I] bf16, box (64, 128), 128B swizzle.
// tm_qi: qI [B, H_I, d_I] bf16 as 3-D (d_I, H_I, B), box (64, npad, 1), 128B swizzle.
cudaError_t launch_indexer_decode(const IndexerArgs& a, const CUtensorMap& tm_ki, const CUtensorMap& tm_qi,
                                  int npad, int num_sms, cudaStream_t stream);

struct PrefillIndexerArgs {
  const float* w;        // [Nq, H_I]
  const int32_t* q_pos;  // [Nq]
  int Nq;
  int S;
  int max_pos;
  int H_I;
  int d_I;
  float* scores;  // [Nq, ld]
  int64_t ld;
  DeviceStatus* status;
};

// Block-of-queries kernel: H_I a power of two in [2, 64], d_I 64 or 128.
bool indexer_prefill_supported(int H_I, int d_I);
// tm_ki: KI [S, d_I], box (64, 128); tm_qi: qI as 2-D [Nq*H_I, d_I], box (64, 256), 128B swizzle.
cudaError_t launch_indexer_prefill(const PrefillIndexerArgs& a, const CUtensorMap& tm_ki,
                                   const CUtensorMap& tm_qi, int num_sms, cudaStream_t stream);

}  // namespace sa
