// Dynamic k by routing mass [CLSA news article, sections "Le cout : limites
// de compatibilite" and "Ce que cela signifie pour l'inference sur longs
// contextes": the indexer layer could choose k per query rather than a fixed
// k; the pages give no rule].  Reading: row q keeps the smallest number m of
// its tokens, in the top-k order (score descending, lower index first),
// whose summed score reaches the fraction tau of the row's total score, but
// at most k_max; a row that never reaches it keeps min(n, k_max).
//
// One CTA per row, after the top-k kernels have selected the row's top
// k_max with their scores (ascending index order):
//   1  the row's total in fp64 (every thread a strided share, block sum);
//   2  the selection as 64-bit keys (order key of the score, then the
//      complemented index) sorted descending in shared memory (bitonic), so
//      position j holds the (j+1)-th token of the top-k order;
//   3  an fp64 prefix sum over the sorted scores; m is one past the first
//      position whose prefix reaches tau * total;
//   4  the selection, still in index order, keeps the entries whose key is
//      at least the m-th key, compacted by a block scan; -1 after them.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "sm100.cuh"
#include "status.cuh"
#include "topk.cuh"

namespace sa {
namespace {

constexpr int kT = 1024;
constexpr int kW = kT / 32;

__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_score(uint64_t key) {
  const uint32_t ok = (uint32_t)(key >> 32);
  return __uint_as_float((ok & 0x80000000u) ? (ok & 0x7FFFFFFFu) : ~ok);
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__global__ void __launch_bounds__(kT) topk_dynamic_kernel(const float* __restrict__ scores, int64_t ld,
                                                          const int32_t* __restrict__ n_valid, int n_max,
                                                          const int32_t* __restrict__ sel_idx,
                                                          const float* __restrict__ sel_s, int k_max, int kp2,
                                                          double tau, int32_t* __restrict__ idx,
                                                          int32_t* __restrict__ counts, DeviceStatus* status) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint64_t* key = reinterpret_cast<uint64_t*>(smem_raw);  // [kp2]
  __shared__ double wsd[kW];
  __shared__ int wsi[kW + 1];
  __shared__ int s_first;
  const int q = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_wait();  // the selection comes from the top-k kernel before this one
  int n = n_valid[q];
  if (n < 0 || n > n_max) {
    if (tid == 0) report(status, kErrDevice, kKernTopk, q, n, n_max);
    n = n < 0 ? 0 : n_max;
  }
  const int m0 = n < k_max ? n : k_max;
  const float* row = scores + (int64_t)q * ld;
  // ---- 1: the row's total score ----
  double part = 0.0;
  for (int t = tid; t < n; t += kT) part += (double)row[t];
  part = warp_sum(part);
  if (lane == 0) wsd[warp] = part;
  // ---- 2: the selection, sorted descending by (score, lower index) ----
  const int32_t* si = sel_idx + (int64_t)q * k_max;
  const float* ss = sel_s + (int64_t)q * k_max;
  for (int j = tid; j < kp2; j += kT)
    key[j] = j < m0 ? ((uint64_t)order_key(ss[j]) << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)si[j]) : 0ull;
  if (tid == 0) s_first = 0x7FFFFFFF;
  __syncthreads();
  double total = 0.0;
  for (int w = 0; w < kW; ++w) total += wsd[w];
  for (int k2 = 2; k2 <= kp2; k2 <<= 1) {
    for (int j = k2 >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < kp2; i += kT) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const uint64_t a = key[i], b = key[ixj];
          const bool desc = (i & k2) == 0;
          if (desc ? (a < b) : (a > b)) {
            key[i] = b;
            key[ixj] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  // ---- 3: running sum in the top-k order, first position reaching the target ----
  // thread t owns positions [t*per, (t+1)*per)
  const int per = kp2 / kT > 0 ? kp2 / kT : 1;
  const int p0 = tid * per;
  double loc = 0.0;
  for (int e = 0; e < per; ++e) {
    const int j = p0 + e;
    if (j < m0) loc += (double)key_score(key[j]);
  }
  double incl = loc;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double x = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += x;
  }
  __syncthreads();
  if (lane == 31) wsd[warp] = incl;
  __syncthreads();
  double before = incl - loc;
  for (int w = 0; w < warp; ++w) before += wsd[w];
  const double target = tau * total;
  double run = before;
  for (int e = 0; e < per; ++e) {
    const int j = p0 + e;
    if (j < m0) {
      run += (double)key_score(key[j]);
      if (run >= target) {
        atomicMin(&s_first, j);
        break;
      }
    }
  }
  __syncthreads();
  const int m = s_first < m0 ? s_first + 1 : m0;
  const uint64_t cut = m > 0 ? key[m - 1] : ~0ull;
  // ---- 4: the kept entries, in index order ----
  int32_t* out = idx + (int64_t)q * k_max;
  int carry = 0;
  for (int base = 0; base < k_max; base += kT) {
    const int j = base + tid;
    bool keep = false;
    int32_t v = -1;
    if (j < m0) {
      v = si[j];
      keep = (((uint64_t)order_key(ss[j]) << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)v)) >= cut;
    }
    const uint32_t bal = __ballot_sync(0xffffffffu, keep);
    if (lane == 0) wsi[warp] = __popc(bal);
    __syncthreads();
    if (warp == 0) {
      const int c = wsi[lane];
      int ci = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, ci, o);
        if (lane >= o) ci += x;
      }
      wsi[lane] = ci - c;
      if (lane == 31) wsi[kW] = ci;
    }
    __syncthreads();
    if (keep) out[carry + wsi[warp] + __popc(bal & ((1u << lane) - 1u))] = v;
    carry += wsi[kW];
    __syncthreads();
  }
  pdl_trigger();
  for (int j = m + tid; j < k_max; j += kT) out[j] = -1;
  if (tid == 0) counts[q] = m;
}

}  // namespace

size_t topk_dynamic_smem_bytes(int k_max) {
  int kp2 = 1;
  while (kp2 < k_max) kp2 <<= 1;
  if (kp2 < kT) kp2 = kT;
  return (size_t)kp2 * 8;
}

cudaError_t launch_topk_dynamic(const float* scores, int64_t ld, const int32_t* n_valid, int Nq, int n_max,
                                const int32_t* sel_idx, const float* sel_s, int k_max, double tau, int32_t* idx,
                                int32_t* counts, DeviceStatus* status, cudaStream_t stream) {
  int kp2 = 1;
  while (kp2 < k_max) kp2 <<= 1;
  if (kp2 < kT) kp2 = kT;
  const size_t smem = (size_t)kp2 * 8;  // at most 32 KB: within the default limit, no attribute needed
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)Nq);
  cfg.blockDim = dim3(kT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, topk_dynamic_kernel, scores, ld, n_valid, n_max, sel_idx, sel_s, k_max, kp2, tau, idx,
                         counts, status);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace sa
