// Launch interface of the sparse attention kernels (internal to libsa).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "status.cuh"

namespace sa {

struct AttnArgs {
  const uint16_t* Q;
  const uint16_t* K;
  const uint16_t* V;
  // decode: keys of (b, g) are idx[b, 0:k]; the cache of sequence b starts at
  // seq_off[b]*Hkv*d and is laid out [Hkv, seq_len[b], d]
  const int64_t* seq_off;
  const int32_t* seq_len;
  const int32_t* idx;
  int k;
  // prefill (prefill != 0): keys of group g are the blocks
  // kv_indices[kv_indptr[g] : kv_indptr[g+1]] of `block` tokens; cache [Hkv, S, d];
  // query p sees keys t <= q_pos[p]
  int prefill;
  const int32_t* q_pos;
  const int32_t* kv_indptr;
  const int32_t* kv_indices;
  int S;
  int block;
  int Nq;

  int L;  // decode: layers in the group
  int B;
  int Hq;
  int Hkv;
  int G;       // Hq / Hkv
  int R;       // query rows per (b, g): L*G (decode) or Nq*G (prefill)
  int n_mtiles;
  int n_split;         // 1, 2, 4 or 8: the splits of a row tile form one cluster
  int keys_per_split;  // multiple of 128
  float scale_log2;    // softmax scale * log2(e)
  void* O;
  int out_f32;
  // partial output (context-parallel decode): when set, O (fp32) receives each
  // row's output before normalisation, relative to the row's reference logit
  // m (log2 units, within 8 of the max), and ml the row's (m, sum of weights)
  float2* ml = nullptr;
  // decode, optional: idx_count[b] entries of idx row b are real, the rest
  // padding; the key splits then cover only those entries
  const int32_t* idx_count = nullptr;
  // CUDA-core path with n_split > 1 key slices: per-(b, g) counters (zero
  // between launches) and the slices' partials [B*Hkv][n_split][rows][d],
  // (m, l) [B*Hkv][n_split][rows]
  uint32_t* small_cnt = nullptr;
  // few-rows path: read idx, seq_off, seq_len, K and V (and start the first
  // loads) before griddepcontrol.wait.  Only when the stream's previous
  // kernel writes none of them and triggers its dependents after its own
  // wait (a launch of this same path).
  int early = 0;
  float* small_po = nullptr;
  float2* small_pml = nullptr;
  // prefill with ordered skipping (osk_order set, n_split 1): row tile mt
  // reads the blocks osk_order[mt*osk_ld + 0 : |T|] in that order, 128 keys
  // (two 64-token blocks) per tile.  After each tile every row's share of
  // its running softmax mass that the tile added is checked; the first tile
  // where every row's share is below osk_tau is followed by the two tiles
  // already in flight and nothing more.  osk_steps[unit] = tiles run.
  const int32_t* osk_order = nullptr;
  int64_t osk_ld = 0;
  float osk_tau = 0.f;
  int32_t* osk_steps = nullptr;
  DeviceStatus* status;
};

int attn_num_units(const AttnArgs& a);
// tm_q / tm_k / tm_v: Q, K, V as 2-D [rows, 128] bf16 tensors, 128-byte
// swizzle.  tm_q, and tm_k / tm_v in decode: box 64 x 1 (rows gathered four at
// a time).  tm_k / tm_v in prefill: box 64 x 64 (one KV block per load).
cudaError_t launch_sparse_attn(const AttnArgs& a, const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                               const CUtensorMap& tm_v, bool precise_p, cudaStream_t stream);

// Path for at most kSmallMaxRows query rows per (b, g) (decode, neither
// partial outputs nor idx_count): warp-level MMA, one CTA per (b, g, key
// slice).  small_attn_splits gives n_split for `units` = B*Hkv (1 when units
// exceeds the counters available); with n_split > 1 the call needs
// small_attn_scratch_bytes of workspace scratch and the counters.
constexpr int kSmallMaxRows = 8;
constexpr int kSmallMaxSplits = 16;
int small_attn_rows(int R);
int small_attn_splits(int units, int k, int sms, int max_counters);
size_t small_attn_scratch_bytes(int units, int ns, int R);
cudaError_t launch_sparse_attn_small(const AttnArgs& a, cudaStream_t stream);

// Path for 9 to kMidMaxRows query rows per (b, g) (decode, neither partial
// outputs nor idx_count): warp-level MMA, one warp per 16 rows, one CTA per
// (b, g, key slice), then (n_split > 1) a merge kernel.  mid_attn_splits
// gives n_split; with n_split > 1 the call needs mid_attn_scratch_bytes of
// workspace scratch for the partials (small_po, small_pml, [B*Hkv][n_split][R]).
constexpr int kMidMaxRows = 128;  // the kernel supports up to this many
constexpr int kMidMaxSplits = 16;
constexpr int kMidMaxSlice = 4096;  // index entries per slice: k <= kMidMaxSplits * kMidMaxSlice
int mid_attn_splits(int units, int R, int k, int sms);
size_t mid_attn_scratch_bytes(int units, int ns, int R);
cudaError_t launch_sparse_attn_mid(const AttnArgs& a, cudaStream_t stream);

}  // namespace sa
