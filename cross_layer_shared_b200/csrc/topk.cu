// Top-k selection over indexer scores.
//
// Definition [IndexCache technical summary section 1: keep the k most
// relevant tokens; CLSA news article "Comment CLSA fonctionne": the top-k
// selection runs once and its index is reused]: for each row, the
// min(k, n) largest scores, ties to the LOWER index, emitted in ascending
// index order and padded with -1.
//
// Radix select on order-preserving 32-bit keys (float bits, sign-flipped;
// -0 mapped to +0).  One CTA of 1024 threads per row.  Every pass over the
// row keeps eight loads per thread in flight.
//   pass 1  histogram of key bits [31:20] over the row          (global)
// Rows of up to 262144 keys whose threshold bucket fits in shared memory:
//   pass 2  keys above the bucket set their bit in a shared bitmap of the
//           row; the bucket's (key, index) pairs go to a shared list (global)
//   smem    digits [19:10], [9:0] (then the index, for ties) fix the k-th
//           key; the kept bucket keys set their bits; the set bits are
//           emitted in index order from one block-wide prefix sum.
// Otherwise:
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
constexpr int kCap = 8192;    // threshold-bucket keys kept in shared memory
constexpr int kBitmapKeys = 262144;  // rows up to this length take the bitmap path
constexpr int kLd = 8;        // loads in flight per thread

__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;  // -0 == +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct Smem {
  uint32_t hist[kBins1];
  uint32_t cand[kCap];
  uint32_t cand_idx[kCap];
  uint32_t bitmap[kBitmapKeys / 32];
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

// Radix select, descending, over the candidate pairs (key, index) in
// shared memory: the need-th largest value of val(j) among those with
// pred(j) whose bits outside the levels equal (prefix, mask).  Returns T;
// *need becomes how many values == T are taken, *n_eq how many equal T.
template <class Val, class Pred>
__device__ uint32_t cand_radix(Smem& sm, int nc, Val val, Pred pred, uint32_t prefix, uint32_t mask,
                               const int* shifts, const int* widths, int nlev, int* need, int* n_eq) {
  for (int lv = 0; lv < nlev; ++lv) {
    const int shift = shifts[lv], nb = 1 << widths[lv];
    for (int i = threadIdx.x; i < nb; i += kThreads) sm.hist[i] = 0;
    __syncthreads();
    for (int j = threadIdx.x; j < nc; j += kThreads) {
      if (!pred(j)) continue;
      const uint32_t v = val(j);
      if ((v & mask) == prefix) atomicAdd(&sm.hist[(v >> shift) & (uint32_t)(nb - 1)], 1u);
    }
    __syncthreads();
    find_bin_desc(sm, sm.hist, nb, *need);
    prefix |= (uint32_t)sm.sel_bin << shift;
    mask |= (uint32_t)(nb - 1) << shift;
    *need -= sm.sel_before;
    *n_eq = (int)sm.hist[sm.sel_bin];
    __syncthreads();
  }
  return prefix;
}

// The rest of a row whose threshold bucket (digit `prefix`, `need` keys of
// it taken) fits in shared memory: one more pass over the row marks the keys
// above the bucket in a bitmap and lists the bucket's keys; the k-th key and
// the lower-index tie rule are settled on the list; the set bits are emitted
// in index order.
__device__ void select_by_bitmap(Smem& sm, const float* __restrict__ row, int n, int k, uint32_t prefix, int need,
                                 int32_t* __restrict__ out, float* __restrict__ out_s) {
  const int tid = threadIdx.x, lane = tid & 31;
  const int nw = (n + 31) >> 5;
  const uint32_t beta = prefix >> 20;
  for (int i = tid; i < nw; i += kThreads) sm.bitmap[i] = 0;
  if (tid == 0) sm.ncand = 0;
  __syncthreads();
  for (int base = 0; base < n; base += kLd * kThreads) {
    uint32_t key[kLd];
#pragma unroll
    for (int u = 0; u < kLd; ++u) {
      const int i = base + u * kThreads + tid;
      key[u] = i < n ? order_key(__ldg(&row[i])) : 0u;
    }
#pragma unroll
    for (int u = 0; u < kLd; ++u) {
      const int i = base + u * kThreads + tid;  // lanes of a warp hold 32 consecutive keys
      const bool in = i < n;
      const uint32_t d = key[u] >> 20;
      const uint32_t above = __ballot_sync(0xffffffffu, in && d > beta);
      const uint32_t eq = __ballot_sync(0xffffffffu, in && d == beta);
      if (lane == 0 && above) sm.bitmap[i >> 5] = above;  // one warp owns the word
      if (eq) {
        int slot = 0;
        if (lane == 0) slot = atomicAdd(&sm.ncand, __popc(eq));
        slot = __shfl_sync(0xffffffffu, slot, 0);
        if ((eq >> lane) & 1u) {
          const int p = slot + __popc(eq & ((1u << lane) - 1u));
          sm.cand[p] = key[u];
          sm.cand_idx[p] = (uint32_t)i;
        }
      }
    }
  }
  __syncthreads();
  const int nc = sm.ncand;
  int n_eq = 0;
  const int ks[2] = {10, 0}, kw[2] = {10, 10};
  const uint32_t T = cand_radix(sm, nc, [&](int j) { return sm.cand[j]; }, [](int) { return true; }, prefix,
                                0xFFF00000u, ks, kw, 2, &need, &n_eq);
  uint32_t cut = 0xFFFFFFFFu;
  if (need < n_eq) {  // the `need` lowest indices among keys == T: largest values of ~index
    int need2 = need, n2 = 0;
    const int is[3] = {21, 10, 0}, iw[3] = {11, 11, 10};
    cut = ~cand_radix(sm, nc, [&](int j) { return ~sm.cand_idx[j]; }, [&](int j) { return sm.cand[j] == T; }, 0u,
                      0u, is, iw, 3, &need2, &n2);
  }
  for (int j = tid; j < nc; j += kThreads) {
    const uint32_t kx = sm.cand[j], ix = sm.cand_idx[j];
    if (kx > T || (kx == T && ix <= cut)) atomicOr(&sm.bitmap[ix >> 5], 1u << (ix & 31));
  }
  __syncthreads();
  // emit: thread t owns words [t*per, t*per + per)
  const int per = (nw + kThreads - 1) / kThreads;
  int cnt = 0;
  for (int j = 0; j < per; ++j) {
    const int wi = tid * per + j;
    if (wi < nw) cnt += __popc(sm.bitmap[wi]);
  }
  int tot;
  int pos = block_exclusive_scan(cnt, sm.warp_sum, &tot);
  for (int j = 0; j < per; ++j) {
    const int wi = tid * per + j;
    if (wi >= nw) break;
    uint32_t x = sm.bitmap[wi];
    while (x) {
      const int b = __ffs(x) - 1;
      x &= x - 1;
      const int i = (wi << 5) + b;
      if (pos < k) {
        out[pos] = i;
        if (out_s) out_s[pos] = row[i];
      }
      ++pos;
    }
  }
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
  for (int base = 0; base < n; base += kLd * kThreads) {
    uint32_t key[kLd];
#pragma unroll
    for (int u = 0; u < kLd; ++u) {
      const int i = base + u * kThreads + tid;
      key[u] = i < n ? order_key(__ldg(&row[i])) : 0u;
    }
#pragma unroll
    for (int u = 0; u < kLd; ++u)
      if (base + u * kThreads + tid < n) atomicAdd(&sm.hist[key[u] >> 20], 1u);
  }
  __syncthreads();
  find_bin_desc(sm, sm.hist, kBins1, k);
  uint32_t prefix = (uint32_t)sm.sel_bin << 20;
  int need = k - sm.sel_before;
  const int bucket = (int)sm.hist[sm.sel_bin];
  __syncthreads();
  if (n <= kBitmapKeys && bucket <= kCap) {
    select_by_bitmap(sm, row, n, k, prefix, need, out, out_s);
    return;
  }

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
