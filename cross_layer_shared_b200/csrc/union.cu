// Block union for chunked prefill [CompactAttention technical summary,
// "Methodologie", selection step]: every selected token t maps to KV block
// t / block; the union runs over all queries of the chunk (Q-block union)
// and over the query heads of each GQA group (intra-group union; the index
// is shared by all heads here, so every group's table is the same set).
// The result is the minimal coverage-preserving table T_g, emitted as CSR
// (kv_indptr, kv_indices) with blocks sorted ascending.
#include <cuda_runtime.h>
#include <stdint.h>

#include "status.cuh"
#include "union.cuh"

namespace sa {
namespace {

// Eight entries per thread are loaded before any is marked, so that a
// thread waits one load latency per eight entries instead of one per entry.
__global__ void union_mark_kernel(const int32_t* __restrict__ idx, int64_t n, int S, int block,
                                  uint8_t* __restrict__ mark, DeviceStatus* status) {
  constexpr int kBatch = 8;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i0 < n; i0 += kBatch * stride) {
    int t[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) t[u] = i0 + u * stride < n ? __ldg(&idx[i0 + u * stride]) : -1;
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      if (t[u] < 0) continue;
      if (t[u] >= S) {
        report(status, kErrDevice, kKernUnion, i0 + u * stride, t[u], S);
        continue;
      }
      mark[t[u] / block] = 1;
    }
  }
}

constexpr int kCompactThreads = 1024;

__device__ int scan_block(int v, int* ws, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
  for (int o = 1; o < 32; o <<= 1) {
    const int x = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += x;
  }
  if (lane == 31) ws[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int w = ws[lane];
    int wi = w;
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += x;
    }
    ws[lane] = wi - w;
    if (lane == 31) ws[32] = wi;
  }
  __syncthreads();
  const int ex = ws[warp] + incl - v;
  *total = ws[32];
  __syncthreads();
  return ex;
}

// One CTA: count the marked blocks, then write the sorted list once per group.
__global__ void __launch_bounds__(kCompactThreads) union_compact_kernel(const uint8_t* __restrict__ mark, int nb,
                                                                        int Hkv, int32_t* __restrict__ kv_indptr,
                                                                        int32_t* __restrict__ kv_indices) {
  __shared__ int ws[33];
  int n = 0;
  for (int base = 0; base < nb; base += kCompactThreads) {
    const int i = base + threadIdx.x;
    const int f = (i < nb && mark[i]) ? 1 : 0;
    int tot;
    scan_block(f, ws, &tot);
    n += tot;
  }
  int pos = 0;
  for (int base = 0; base < nb; base += kCompactThreads) {
    const int i = base + threadIdx.x;
    const int f = (i < nb && mark[i]) ? 1 : 0;
    int tot;
    const int ex = scan_block(f, ws, &tot);
    if (f)
      for (int g = 0; g < Hkv; ++g) kv_indices[(int64_t)g * n + pos + ex] = i;
    pos += tot;
  }
  for (int g = threadIdx.x; g <= Hkv; g += kCompactThreads) kv_indptr[g] = g * n;
}

}  // namespace

cudaError_t launch_block_union(const int32_t* idx, int Nq, int k, int S, int block, int Hkv, uint8_t* mark,
                               int32_t* kv_indptr, int32_t* kv_indices, DeviceStatus* status,
                               cudaStream_t stream) {
  const int nb = (S + block - 1) / block;
  cudaError_t e = cudaMemsetAsync(mark, 0, (size_t)nb, stream);
  if (e != cudaSuccess) return e;
  const int64_t n = (int64_t)Nq * k;
  if (n > 0) {
    int blocks = (int)((n + 255) / 256);
    if (blocks > 148 * 8) blocks = 148 * 8;
    union_mark_kernel<<<blocks, 256, 0, stream>>>(idx, n, S, block, mark, status);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  union_compact_kernel<<<1, kCompactThreads, 0, stream>>>(mark, nb, Hkv, kv_indptr, kv_indices);
  return cudaGetLastError();
}

}  // namespace sa
