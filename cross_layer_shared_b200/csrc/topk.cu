// Top-k selection over indexer scores.
//
// Definition [IndexCache technical summary section 1: keep the k most
// relevant tokens; CLSA news article "Comment CLSA fonctionne": the top-k
// selection runs once and its index is reused]: for each row, the
// min(k, n) largest scores, ties to the LOWER index, emitted in ascending
// index order and padded with -1.
//
// Radix select on order-preserving 32-bit keys (float bits, sign-flipped;
// -0 mapped to +0).  One CTA of 1024 threads per row:
//   pass 1  histogram of key bits [31:20] over the row          (global)
//   pass 2  collect the keys of the threshold bucket into smem  (global)
//           (or, if that bucket is too large, histogram passes in global)
//   smem    digits [19:10] and [9:0] fix the k-th key T and how many keys
//           equal to T are needed
//   pass 3  (only if some keys equal T must be dropped) find, in index
//           order, the last index among keys == T that is kept
//   pass 4  emit, in index order, every key > T and the kept keys == T,
//           positions from a block-wide prefix sum (warp ballots)
// Every comparison is on integer keys, so the set is exact and unique.
#include <cuda_runtime.h>
#include <stdint.h>

#include "sm100.cuh"
#include "status.cuh"
#include "topk.cuh"

namespace sa {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kBins1 = 4096;  // bits [31:20]
constexpr int kBins2 = 1024;  // bits [19:10] and [9:0]
constexpr int kCap = 16384;   // threshold-bucket keys kept in shared memory

__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;  // -0 == +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct Smem {
  uint32_t hist[kBins1];
  uint32_t cand[kCap];
  int warp_sum[kWarps + 1];
  int ncand;
  int sel_bin;
  int sel_before;
  int cut;
};

// Block-wide exclusive prefix sum of one int per thread; also returns the total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_sum, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int x = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += x;
  }
  __syncthreads();
  if (lane == 31) warp_sum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = lane < kWarps ? warp_sum[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += x;
    }
    if (lane < kWarps) warp_sum[lane] = wi - w;  // exclusive per warp
    if (lane == kWarps - 1) warp_sum[kWarps] = wi;
  }
  __syncthreads();
  const int excl = warp_sum[warp] + incl - v;
  *total = warp_sum[kWarps];
  __syncthreads();
  return excl;
}

// Scans hist[0..nb) from the top bin down; finds the bin where the running
// count reaches `need` (1 <= need <= sum).  Writes sel_bin and sel_before
// (count in bins strictly above it).
__device__ void find_bin_desc(Smem& sm, const uint32_t* hist, int nb, int need) {
  const int per = (nb + kThreads - 1) / kThreads;
  // thread i owns bins [nb-1-i*per, nb-1-(i+1)*per) in descending order
  int local = 0;
  for (int j = 0; j < per; ++j) {
    const int bin = nb - 1 - (threadIdx.x * per + j);
    if (bin >= 0) local += (int)hist[bin];
  }
  int total;
  int before = block_exclusive_scan(local, sm.warp_sum, &total);
  if (before < need && need <= before + local) {
    for (int j = 0; j < per; ++j) {
      const int bin = nb - 1 - (threadIdx.x * per + j);
      if (bin < 0) break;
      const int c = (int)hist[bin];
      if (before + c >= need) {
        sm.sel_bin = bin;
        sm.sel_before = before;
        break;
      }
      before += c;
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kThreads, 1)
topk_rows_kernel(const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ n_valid, int n_max,
                 int k, int32_t* __restrict__ idx, float* __restrict__ top_scores, DeviceStatus* status) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
  const int q = blockIdx.x;
  const int tid = threadIdx.x;
  const float* row = scores + (int64_t)q * ld;
  int32_t* out = idx + (int64_t)q * k;
  float* out_s = top_scores ? top_scores + (int64_t)q * k : nullptr;

  int n = n_valid[q];
  if (n < 0 || n > n_max) {
    if (tid == 0) report(status, kErrDevice, kKernTopk, q, n, n_max);
    n = n < 0 ? 0 : n_max;
  }
  if (n <= k) {
    for (int i = tid; i < k; i += kThreads) {
      out[i] = i < n ? i : -1;
      if (out_s) out_s[i] = i < n ? row[i] : 0.f;
    }
    return;
  }

  // ---- pass 1: top 12 bits ---------------------------------------------
  for (int i = tid; i < kBins1; i += kThreads) sm.hist[i] = 0;
  if (tid == 0) sm.ncand = 0;
  __syncthreads();
  for (int i = tid; i < n; i += kThreads) atomicAdd(&sm.hist[order_key(row[i]) >> 20], 1u);
  __syncthreads();
  find_bin_desc(sm, sm.hist, kBins1, k);
  uint32_t prefix = (uint32_t)sm.sel_bin << 20;
  int need = k - sm.sel_before;
  const int bucket = (int)sm.hist[sm.sel_bin];
  __syncthreads();

  // ---- digits [19:10] and [9:0] ------------------------------------------
  if (bucket <= kCap) {
    for (int i = tid; i < n; i += kThreads) {
      const uint32_t key = order_key(row[i]);
      if ((key >> 20) == (prefix >> 20)) sm.cand[atomicAdd(&sm.ncand, 1)] = key;
    }
    __syncthreads();
    const int nc = sm.ncand;
    for (int lvl = 0; lvl < 2; ++lvl) {
      const int shift = lvl == 0 ? 10 : 0;
      const uint32_t hi_mask = lvl == 0 ? 0xFFF00000u : 0xFFFFFC00u;
      for (int i = tid; i < kBins2; i += kThreads) sm.hist[i] = 0;
      __syncthreads();
      for (int i = tid; i < nc; i += kThreads) {
        const uint32_t key = sm.cand[i];
        if ((key & hi_mask) == prefix) atomicAdd(&sm.hist[(key >> shift) & 1023u], 1u);
      }
      __syncthreads();
      find_bin_desc(sm, sm.hist, kBins2, need);
      prefix |= (uint32_t)sm.sel_bin << shift;
      need -= sm.sel_before;
      __syncthreads();
    }
  } else {
    for (int lvl = 0; lvl < 2; ++lvl) {
      const int shift = lvl == 0 ? 10 : 0;
      const uint32_t hi_mask = lvl == 0 ? 0xFFF00000u : 0xFFFFFC00u;
      for (int i = tid; i < kBins2; i += kThreads) sm.hist[i] = 0;
      __syncthreads();
      for (int i = tid; i < n; i += kThreads) {
        const uint32_t key = order_key(row[i]);
        if ((key & hi_mask) == prefix) atomicAdd(&sm.hist[(key >> shift) & 1023u], 1u);
      }
      __syncthreads();
      find_bin_desc(sm, sm.hist, kBins2, need);
      prefix |= (uint32_t)sm.sel_bin << shift;
      need -= sm.sel_before;
      __syncthreads();
    }
  }
  const uint32_t T = prefix;          // the k-th largest key
  const int n_eq = (int)sm.hist[T & 1023u];  // keys equal to T
  // `need` keys equal to T are kept: the lowest-index ones

  // ---- pass 3: last kept index among keys == T ---------------------------
  int cut = 0x7FFFFFFF;
  if (need < n_eq) {
    int seen = 0;
    for (int base = 0; base < n; base += kThreads) {
      const int i = base + tid;
      const int f = (i < n && order_key(row[i]) == T) ? 1 : 0;
      int tot;
      const int ex = block_exclusive_scan(f, sm.warp_sum, &tot);
      if (f && seen + ex + 1 == need) sm.cut = i;
      seen += tot;
      __syncthreads();
      if (seen >= need) break;
    }
    cut = sm.cut;
  }

  // ---- pass 4: emit in index order --------------------------------------
  int written = 0;
  for (int base = 0; base < n && written < k; base += kThreads) {
    const int i = base + tid;
    int f = 0;
    float v = 0.f;
    if (i < n) {
      v = row[i];
      const uint32_t key = order_key(v);
      f = (key > T || (key == T && i <= cut)) ? 1 : 0;
    }
    int tot;
    const int ex = block_exclusive_scan(f, sm.warp_sum, &tot);
    if (f) {
      const int pos = written + ex;
      if (pos < k) {
        out[pos] = i;
        if (out_s) out_s[pos] = v;
      }
    }
    written += tot;
  }
}

}  // namespace

size_t topk_rows_smem_bytes() { return sizeof(Smem) + 16; }

cudaError_t launch_topk_rows(const float* scores, int64_t ld, const int32_t* n_valid, int Nq, int n_max, int k,
                             int32_t* idx, float* top_scores, DeviceStatus* status, cudaStream_t stream) {
  const size_t smem = topk_rows_smem_bytes();
  cudaError_t e = ensure_smem(topk_rows_kernel, smem);
  if (e != cudaSuccess) return e;
  topk_rows_kernel<<<Nq, kThreads, smem, stream>>>(scores, ld, n_valid, n_max, k, idx, top_scores, status);
  return cudaGetLastError();
}

}  // namespace sa
