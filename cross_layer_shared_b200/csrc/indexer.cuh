// Launch interface of the indexer kernels (internal to libsa).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "status.cuh"

namespace sa {

// The new token of every sequence (position seq_len[b] - 1), written into
// the caches by the decode indexer and scored from its fresh indexer key.
// All pointers null: no append.
struct AppendArgs {
  const uint16_t* qI;      // [B, H_I, d_I]: the queries, for the new token's score
  const uint16_t* new_KI;  // [B, d_I]
  uint16_t* KI;            // the indexer-key cache (rows packed by seq_off)
  const uint16_t* new_K;   // [B, Hkv, d] (may be null: no K/V append)
  const uint16_t* new_V;
  uint16_t* K;             // the KV cache: sequence b at seq_off[b]*Hkv*d, [Hkv, seq_len[b], d]
  uint16_t* V;
  int Hkv;
  int d;
};

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
  AppendArgs ap;
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
