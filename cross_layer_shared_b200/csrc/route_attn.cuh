// Launch interface of the indexer-layer attention kernels (internal to libsa).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "status.cuh"

namespace sa {

constexpr int kRouteChunk = 2048;  // keys of one (sequence, KV head) per partial CTA

struct RouteArgs {
  const uint16_t* Q;  // [B, Hq, 128] bf16: the indexer layer's queries
  const uint16_t* K;  // sequence b at row seq_off[b]*Hkv, [Hkv, seq_len[b], 128]
  const uint16_t* V;
  const int64_t* seq_off;
  const int32_t* seq_len;
  int B, Hq, Hkv, S_max;
  int64_t n_tokens;
  float scale_log2;  // softmax scale * log2(e)
  int n_split;       // ceil(S_max / kRouteChunk)
  int64_t zld;       // row stride of z (floats)
  float* z;          // [B, Hq, zld] logits in log2 units (scratch)
  float2* part_ml;   // [B, Hq, n_split] (chunk max, sum of 2^(z - max))
  float* part_o;     // [B, Hq, n_split, 128] sum of 2^(z - max) V
  float* scores;     // [B, ld] routing scores (sum over heads of the attention weights)
  int64_t ld;
  void* O;           // [B, Hq, 128] dense output, bf16 or fp32
  int out_f32;
  DeviceStatus* status;
};

size_t route_ws_bytes(int B, int S_max, int Hq);  // scratch after the workspace header
// tm_k / tm_v: the packed K / V caches as 2-D [n_tokens*Hkv, 128] bf16, box 64
// x 128 rows, 128-byte swizzle; tm_q: Q as 3-D (128, Hq, B), box (64, 16, 1).
cudaError_t launch_indexer_layer_attn(const RouteArgs& a, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                                      const CUtensorMap& tm_q, cudaStream_t stream);

}  // namespace sa
