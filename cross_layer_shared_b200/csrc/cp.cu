// Context-parallel decode: the pieces around the shared-index path when every
// rank holds a contiguous slice of each sequence's context (rank r the
// tokens [lo_r(b), hi_r(b)), slices in rank order).
//
// A step on rank r: its indexer scores and top-k (with scores) over its
// slice; the candidates of all ranks exchanged; cp_gather_kernel, the top-k
// and cp_local_kernel below keep this rank's share of the global top-k;
// attention over its selected rows with partial outputs (m, l, o before
// normalisation); the partials exchanged; combine_partials_kernel merges
// them.  The result equals the single-GPU step: a
// token of the global top-k is in its slice's top-k, ties go to the lower
// index in both (the gathered candidate order, rank-major then ascending
// local index, is ascending global index), and softmax attention over a
// union of disjoint key sets is the log-sum-exp merge of the parts.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "cp.cuh"

namespace sa {
namespace {

// Rank r's [B][k] candidates (at r*stride) -> [B][N*k] rows for the top-k;
// padding (-1) scores -inf; n_valid[b] = N*k.
__global__ void cp_gather_kernel(const float* __restrict__ cand_scores, const int32_t* __restrict__ cand_idx,
                                 int64_t stride, int N, int B, int k, float* __restrict__ rows,
                                 int32_t* __restrict__ n_valid) {
  const int64_t total = (int64_t)N * B * k;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t in_rank = e % ((int64_t)B * k);  // b*k + j
    const int r = (int)(e / ((int64_t)B * k));
    const int b = (int)(in_rank / k);
    const int j = (int)(in_rank % k);
    const int64_t src = r * stride + in_rank;
    rows[((int64_t)b * N + r) * k + j] = cand_idx[src] >= 0 ? cand_scores[src] : -INFINITY;
  }
  for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < B; b += gridDim.x * blockDim.x) n_valid[b] = N * k;
}

// One CTA per sequence: the selected candidate positions (ascending, -1
// padded) that fall in this rank's block [rank*k, rank*k + k) form one run
// of the selection; entry j of the run becomes local entry j - lo, where lo
// counts the selected positions before the block.  The rank's padding
// candidates (-1) sort last in its block, so its real entries lead the run:
// local_idx gets them in order, then -1, and count[b] their number.
__global__ void __launch_bounds__(256) cp_local_kernel(const int32_t* __restrict__ sel,
                                                       const int32_t* __restrict__ cand_idx, int64_t stride, int k,
                                                       int rank, int32_t* __restrict__ local_idx,
                                                       int32_t* __restrict__ count) {
  __shared__ int red[2][8];
  const int b = blockIdx.x;
  const int64_t blo = (int64_t)rank * k, bhi = blo + k;
  const int32_t* srow = sel + (int64_t)b * k;
  const int32_t* crow = cand_idx + rank * stride + (int64_t)b * k;
  int before = 0, valid = 0;
  for (int j = threadIdx.x; j < k; j += blockDim.x) {
    const int p = __ldg(srow + j);
    if (p >= 0 && p < blo) ++before;
    if (p >= blo && p < bhi && __ldg(crow + (p - blo)) >= 0) ++valid;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    before += __shfl_xor_sync(0xffffffffu, before, o);
    valid += __shfl_xor_sync(0xffffffffu, valid, o);
  }
  if ((threadIdx.x & 31) == 0) {
    red[0][threadIdx.x >> 5] = before;
    red[1][threadIdx.x >> 5] = valid;
  }
  __syncthreads();
  int lo = 0, n = 0;
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    lo += red[0][w];
    n += red[1][w];
  }
  int32_t* out = local_idx + (int64_t)b * k;
  for (int j = threadIdx.x; j < k; j += blockDim.x) {
    const int p = __ldg(srow + j);
    if (p >= blo && p < bhi) {
      const int v = __ldg(crow + (p - blo));
      if (v >= 0) out[j - lo] = v;
    }
    if (j >= n) out[j] = -1;
  }
  if (count != nullptr && threadIdx.x == 0) count[b] = n;
}

// One warp per row: o = sum_p 2^(m_p - M) o_p / sum_p 2^(m_p - M) l_p; part p
// at parts + p*o_stride floats and ml + p*ml_stride pairs.
__global__ void combine_partials_kernel(const float* __restrict__ parts, int64_t o_stride,
                                        const float2* __restrict__ ml, int64_t ml_stride, int P, int64_t rows,
                                        float* __restrict__ out_f32, uint16_t* __restrict__ out_bf16) {
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float M = -INFINITY;
  for (int p = 0; p < P; ++p) {
    const float2 v = ml[p * ml_stride + row];
    if (v.y > 0.f) M = fmaxf(M, v.x);
  }
  float L = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (M != -INFINITY) {
    for (int p = 0; p < P; ++p) {
      const float2 v = ml[p * ml_stride + row];
      if (!(v.y > 0.f)) continue;
      const float w = exp2f(v.x - M);
      L += w * v.y;
      const float4 o = reinterpret_cast<const float4*>(parts + p * o_stride + row * 128)[lane];
      acc.x += w * o.x;
      acc.y += w * o.y;
      acc.z += w * o.z;
      acc.w += w * o.w;
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  const float4 f = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  if (out_f32) {
    reinterpret_cast<float4*>(out_f32 + row * 128)[lane] = f;
  } else {
    const uint32_t lo = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f.x)) |
                        ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f.y)) << 16);
    const uint32_t hi = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f.z)) |
                        ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f.w)) << 16);
    reinterpret_cast<uint2*>(out_bf16 + row * 128)[lane] = make_uint2(lo, hi);
  }
}

}  // namespace

cudaError_t launch_cp_gather(const float* cand_scores, const int32_t* cand_idx, int64_t stride, int N, int B, int k,
                             float* rows, int32_t* n_valid, cudaStream_t stream) {
  const int64_t total = (int64_t)N * B * k;
  const int grid = (int)((total + 255) / 256 < 4096 ? (total + 255) / 256 : 4096);
  cp_gather_kernel<<<grid > 0 ? grid : 1, 256, 0, stream>>>(cand_scores, cand_idx, stride, N, B, k, rows,
                                                            n_valid);
  return cudaGetLastError();
}

cudaError_t launch_cp_local(const int32_t* sel, const int32_t* cand_idx, int64_t stride, int B, int k, int rank,
                            int32_t* local_idx, int32_t* count, cudaStream_t stream) {
  cp_local_kernel<<<B, 256, 0, stream>>>(sel, cand_idx, stride, k, rank, local_idx, count);
  return cudaGetLastError();
}

cudaError_t launch_combine_partials(const float* parts, int64_t o_stride, const float2* ml, int64_t ml_stride, int P,
                                    int64_t rows, void* O, bool out_f32, cudaStream_t stream) {
  const int64_t grid = (rows + 7) / 8;
  combine_partials_kernel<<<(unsigned)grid, 256, 0, stream>>>(parts, o_stride, ml, ml_stride, P, rows,
                                                               out_f32 ? static_cast<float*>(O) : nullptr,
                                                               out_f32 ? nullptr : static_cast<uint16_t*>(O));
  return cudaGetLastError();
}

}  // namespace sa
