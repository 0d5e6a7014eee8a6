// Priority list of the union blocks per query block [CoSA lay summary: the
// kernel-aware proxy hands the kernel a priority list, most important block
// first, instead of a yes/no list].  The pages give no priority formula; the
// one built here reuses the indexer's selection: block B's priority for
// query block i is its hit count, the number of index entries of the block's
// queries that fall in B.  The union table T (ascending block ids, the same
// set for every KV group) is ordered by hit count, larger first, equal counts
// by ascending block id.
//
// One CTA per query block: the hit counts go to a shared-memory histogram
// over the KV blocks, each table entry becomes one 64-bit key
// (~count << 32 | id), and a bitonic sort in shared memory orders the keys.
#include <cuda_runtime.h>
#include <stdint.h>

#include "sm100.cuh"
#include "status.cuh"
#include "union.cuh"

namespace sa {
namespace {

constexpr int kKapThreads = 1024;

__global__ void __launch_bounds__(kKapThreads)
kap_order_kernel(const int32_t* __restrict__ idx, int Nq, int k, int S, int block, int q_block, int nb,
                 const int32_t* __restrict__ kv_indptr, const int32_t* __restrict__ kv_indices,
                 int32_t* __restrict__ order, int64_t ld, DeviceStatus* status) {
  extern __shared__ uint64_t kap_smem[];
  const int tid = threadIdx.x;
  const int i = blockIdx.x;
  // a table longer than the KV blocks (or negative) is reported and clamped:
  // the shared-memory key array is sized for at most nb entries
  int nT = kv_indptr[1] - kv_indptr[0];
  if (nT < 0 || nT > nb) {
    if (tid == 0) report(status, kErrDevice, kKernUnion, -1, nT, nb);
    nT = nT < 0 ? 0 : nb;
  }
  const int32_t* T = kv_indices + kv_indptr[0];
  int np = 1;
  while (np < nT) np <<= 1;
  uint64_t* keys = kap_smem;                                    // [np]
  uint32_t* cnt = reinterpret_cast<uint32_t*>(kap_smem + np);  // [nb]
  for (int b = tid; b < nb; b += kKapThreads) cnt[b] = 0;
  __syncthreads();
  const int p0 = i * q_block;
  const int p1 = min(Nq, p0 + q_block);
  const int64_t n = (int64_t)(p1 - p0) * k;
  const int32_t* rows = idx + (int64_t)p0 * k;
  // eight coalesced loads in flight per thread before the atomics
  constexpr int kBatch = 8;
  for (int64_t e0 = tid; e0 < n; e0 += (int64_t)kBatch * kKapThreads) {
    int t[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int64_t e = e0 + (int64_t)u * kKapThreads;
      t[u] = e < n ? __ldg(&rows[e]) : -1;
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u)
      if (t[u] >= 0 && t[u] < S) atomicAdd(&cnt[t[u] / block], 1u);
  }
  __syncthreads();
  for (int j = tid; j < np; j += kKapThreads) {
    uint64_t key = ~0ull;
    if (j < nT) {
      const int b = T[j];
      uint32_t c = 0;
      if (b >= 0 && b < nb) {
        c = cnt[b];
      } else {
        report(status, kErrDevice, kKernUnion, j, b, nb);
      }
      key = ((uint64_t)(~c) << 32) | (uint32_t)b;
    }
    keys[j] = key;
  }
  __syncthreads();
  // bitonic sort, ascending
  for (int size = 2; size <= np; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int j = tid; j < np; j += kKapThreads) {
        const int partner = j ^ stride;
        if (partner > j) {
          const uint64_t x = keys[j], y = keys[partner];
          const bool up = (j & size) == 0;
          if ((x > y) == up) {
            keys[j] = y;
            keys[partner] = x;
          }
        }
      }
      __syncthreads();
    }
  }
  int32_t* out = order + (int64_t)i * ld;
  for (int j = tid; j < nT; j += kKapThreads) out[j] = (int32_t)(uint32_t)(keys[j] & 0xffffffffu);
}

}  // namespace

size_t kap_order_smem(int nb) {
  size_t np = 1;
  while (np < (size_t)nb) np <<= 1;
  return np * 8 + (size_t)nb * 4;
}

cudaError_t launch_kap_order(const int32_t* idx, int Nq, int k, int S, int block, int q_block,
                             const int32_t* kv_indptr, const int32_t* kv_indices, int32_t* order, int64_t ld,
                             DeviceStatus* status, cudaStream_t stream) {
  const int nb = (S + block - 1) / block;
  const int n_qb = (Nq + q_block - 1) / q_block;
  if (n_qb == 0) return cudaSuccess;
  const size_t smem = kap_order_smem(nb);
  cudaError_t e = ensure_smem(kap_order_kernel, smem);
  if (e != cudaSuccess) return e;
  kap_order_kernel<<<n_qb, kKapThreads, smem, stream>>>(idx, Nq, k, S, block, q_block, nb, kv_indptr, kv_indices,
                                                       order, ld, status);
  return cudaGetLastError();
}

}  // namespace sa
