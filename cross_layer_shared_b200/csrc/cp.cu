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
#include "sm100.cuh"
#include "status.cuh"

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


// ---------------------------------------------------------------- radix exchange
// The global top-k by exchanging histograms instead of candidates.  Scores
// map to 32-bit keys that order like the floats (-0 == +0); the k-th largest
// key T is found digit by digit, 12 + 12 + 8 bits, from the histograms of
// every rank (summed on every rank alike):
//   level 0: digit key[31:20] of every local key;
//   level 1: digit key[19:8] of the local keys whose key[31:20] is the
//            level-0 threshold digit;
//   level 2: digit key[7:0] of the keys matching the 24-bit prefix.
// The threshold digit of a level is the one where the count of larger keys,
// summed over the ranks, first reaches the number still needed.  After
// level 2 the prefix is T itself: a rank keeps its keys above T, and of its
// keys equal to T the ones the lower-index rule gives it: ties go to lower
// global indices, that is, to lower ranks first (slices are in rank order),
// then to lower local indices.  When all ranks together hold no more than k
// valid keys, every one is kept.

constexpr int kRadixThreads = 1024;
constexpr int kRadixBins = 4096;
constexpr int kPer = 16;  // entries per thread per round

__device__ __forceinline__ uint32_t cp_order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;  // -0 == +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ int level_bins(int level) { return level == 2 ? 256 : kRadixBins; }

// digit of `key` at `level`, or -1 if key does not match the prefix found so far
__device__ __forceinline__ int level_digit(uint32_t key, int level, uint32_t prefix) {
  if (level == 0) return (int)(key >> 20);
  if (level == 1) return (key >> 20) == prefix ? (int)((key >> 8) & 0xFFFu) : -1;
  return (key >> 8) == prefix ? (int)(key & 0xFFu) : -1;
}

struct RadixSmem {
  int hist[kRadixBins];
  int wsum[kRadixThreads / 32 + 1];
  CpRadixState st;
};

// Block-wide: exclusive prefix sum of v over the CTA's threads in thread order.
__device__ __forceinline__ int block_exclusive_scan(int v, int* wsum, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  __syncthreads();
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  if (warp == 0) {
    const int w = lane < kRadixThreads / 32 ? wsum[lane] : 0;
    int z = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, z, o);
      if (lane >= o) z += y;
    }
    wsum[lane] = z - w;
    if (lane == 31) wsum[kRadixThreads / 32] = z;
  }
  __syncthreads();
  total = wsum[kRadixThreads / 32];
  return wsum[warp] + x - v;
}

// The threshold digit of the previous level from every rank's histogram of
// it (gathered [N] blocks of [B][bins] ints, rank_stride ints apart): the
// digit where the keys above, summed over the ranks, are fewer than the
// number needed and the keys above and at it are not; st.prefix grows by
// that digit and st.need drops by the count above it.  Fewer keys than
// needed in all: st.all = 1.  Also returns, through *at_digit, the digit.
__device__ void radix_threshold(const int32_t* __restrict__ gathered, int64_t rank_stride, int N, int b, int bins,
                                RadixSmem& sm, int* at_digit) {
  {
    // this thread's (up to) 4 digits of every rank: all loads independent
    int acc[4] = {0, 0, 0, 0};
#pragma unroll 4
    for (int r = 0; r < N; ++r) {
      const int32_t* g = gathered + r * rank_stride + (int64_t)b * bins;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = threadIdx.x + u * kRadixThreads;
        if (i < bins) acc[u] += __ldcg(&g[i]);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = threadIdx.x + u * kRadixThreads;
      if (i < bins) sm.hist[i] = acc[u];
    }
  }
  __syncthreads();
  // thread j owns the digits bins-1-per*j .. bins-per*(j+1) (descending)
  const int per = bins / kRadixThreads > 0 ? bins / kRadixThreads : 1;
  const int j0 = threadIdx.x * per;
  int mine = 0;
  for (int u = 0; u < per; ++u)
    if (j0 + u < bins) mine += sm.hist[bins - 1 - (j0 + u)];
  int total = 0;
  int above = block_exclusive_scan(mine, sm.wsum, total);
  const int need = sm.st.need;
  __syncthreads();
  if (total < need) {
    if (threadIdx.x == 0) {
      sm.st.all = 1;
      *at_digit = -1;
    }
  } else {
    for (int u = 0; u < per && j0 + u < bins; ++u) {
      const int dgt = bins - 1 - (j0 + u);
      const int c = sm.hist[dgt];
      if (above < need && above + c >= need) {  // exactly one thread, one digit
        sm.st.prefix = (sm.st.prefix << (bins == 256 ? 8 : 12)) | (uint32_t)dgt;
        sm.st.need = need - above;
        *at_digit = dgt;
      }
      above += c;
    }
  }
  __syncthreads();
}

// One CTA per sequence: the threshold of level-1 (if level > 0), then this
// rank's histogram of level `level` into hist_out [B][bins].
__global__ void __launch_bounds__(kRadixThreads) cp_radix_level_kernel(
    const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ n_local, int k, int N, int level,
    const int32_t* __restrict__ gathered, int64_t rank_stride, CpRadixState* __restrict__ state,
    int32_t* __restrict__ hist_out, DeviceStatus* status) {
  __shared__ RadixSmem sm;
  __shared__ int digit;
  const int b = blockIdx.x, lane = threadIdx.x & 31;
  pdl_wait();
  const int n_raw = __ldcg(&n_local[b]);
  const int n = n_raw > 0 ? n_raw : 0;
  const float* row = scores + (int64_t)b * ld;
  // the first round's scores travel while the threshold is found
  float v[kPer];
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int i = u * kRadixThreads + threadIdx.x;
    v[u] = i < n ? __ldcg(&row[i]) : 0.f;
  }
  if (threadIdx.x == 0) {
    if (level == 0) {
      sm.st.prefix = 0;
      sm.st.need = k;
      sm.st.all = 0;
      sm.st.pad = 0;
    } else {
      sm.st = state[b];
    }
  }
  __syncthreads();
  if (level > 0 && !sm.st.all) radix_threshold(gathered, rank_stride, N, b, kRadixBins, sm, &digit);
  const int bins = level_bins(level);
  for (int i = threadIdx.x; i < bins; i += kRadixThreads) sm.hist[i] = 0;
  __syncthreads();
  pdl_trigger();
  if (n_raw < 0 && threadIdx.x == 0) report(status, kErrDevice, kKernCp, b, n_raw, 0);
  if (!sm.st.all) {
    const uint32_t prefix = sm.st.prefix;
    for (int base = 0; base < n; base += kRadixThreads * kPer) {
      if (base > 0) {
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
          const int i = base + u * kRadixThreads + threadIdx.x;
          v[u] = i < n ? __ldcg(&row[i]) : 0.f;
        }
      }
#pragma unroll
      for (int u = 0; u < kPer; ++u) {
        const int i = base + u * kRadixThreads + threadIdx.x;
        const int dgt = i < n ? level_digit(cp_order_key(v[u]), level, prefix) : -1;
        // scores of one row share their top digits: when the whole warp
        // holds one digit, one atomic adds it (same-address atomics
        // serialise); otherwise each lane adds its own
        const int d0 = __shfl_sync(0xffffffffu, dgt, 0);
        if (__all_sync(0xffffffffu, dgt == d0)) {
          if (lane == 0 && d0 >= 0) atomicAdd(&sm.hist[d0], 32);
        } else if (dgt >= 0) {
          atomicAdd(&sm.hist[dgt], 1);
        }
      }
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < bins; i += kRadixThreads) hist_out[(int64_t)b * bins + i] = sm.hist[i];
  if (threadIdx.x == 0) state[b] = sm.st;
}

// One CTA per sequence: the level-2 threshold, then this rank's entries of
// the global top-k as ascending local indices (then -1) and their count.
__global__ void __launch_bounds__(kRadixThreads) cp_radix_finish_kernel(
    const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ n_local, int k, int N, int rank,
    const int32_t* __restrict__ gathered, int64_t rank_stride, const CpRadixState* __restrict__ state,
    int32_t* __restrict__ local_idx, int32_t* __restrict__ count, DeviceStatus* status) {
  __shared__ RadixSmem sm;
  __shared__ int digit;
  __shared__ int take;
  const int b = blockIdx.x;
  pdl_wait();
  const int n_raw = __ldcg(&n_local[b]);
  const int n = n_raw > 0 ? n_raw : 0;
  const float* row = scores + (int64_t)b * ld;
  // a round: warp w owns the 32*kPer consecutive entries base + w*32*kPer ..,
  // entry u*32 + lane of them in lane `lane` (coalesced loads; (u, lane)
  // order within a warp, warp order across, is index order).  The first
  // round's scores travel while the threshold is found.
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t lt = (1u << lane) - 1u;
  float v[kPer];
  {
    const int w0 = warp * 32 * kPer + lane;
#pragma unroll
    for (int u = 0; u < kPer; ++u) v[u] = w0 + u * 32 < n ? __ldcg(&row[w0 + u * 32]) : 0.f;
  }
  if (threadIdx.x == 0) {
    sm.st = state[b];
    digit = -1;
    take = 0;
  }
  __syncthreads();
  if (!sm.st.all) radix_threshold(gathered, rank_stride, N, b, 256, sm, &digit);
  const bool all = sm.st.all != 0;
  const uint32_t T = sm.st.prefix;  // the k-th largest key (when not all)
  if (!all) {
    // ties at T: the ranks before this one take theirs first (every rank's
    // count at the digit, loaded in parallel)
    if (threadIdx.x < N) sm.hist[threadIdx.x] = __ldcg(&gathered[threadIdx.x * rank_stride + (int64_t)b * 256 + digit]);
    __syncthreads();
    if (threadIdx.x == 0) {
      int before = 0;
      for (int r = 0; r < rank; ++r) before += sm.hist[r];
      const int t = sm.st.need - before, mine = sm.hist[rank];
      take = t < 0 ? 0 : (t > mine ? mine : t);
    }
  }
  __syncthreads();
  pdl_trigger();
  if (n_raw < 0 && threadIdx.x == 0) report(status, kErrDevice, kKernCp, b, n_raw, 0);
  int32_t* out = local_idx + (int64_t)b * k;
  int kept = 0, ties = 0;  // before this round
  const int take_t = take;
  for (int base = 0; base < n; base += kRadixThreads * kPer) {
    const int w0 = base + warp * 32 * kPer + lane;
    if (base > 0) {
#pragma unroll
      for (int u = 0; u < kPer; ++u) v[u] = w0 + u * 32 < n ? __ldcg(&row[w0 + u * 32]) : 0.f;
    }
    uint32_t gtb[kPer], eqb[kPer];  // warp-uniform masks per u
    int weq = 0;
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      bool g = false, e = false;
      if (w0 + u * 32 < n) {
        const uint32_t key = cp_order_key(v[u]);
        g = all || key > T;
        e = !all && key == T;
      }
      gtb[u] = __ballot_sync(0xffffffffu, g);
      eqb[u] = __ballot_sync(0xffffffffu, e);
      weq += __popc(eqb[u]);
    }
    // ties before this warp (this round), then each lane's tie ordinal
    int tot_eq = 0;
    const int eq_scan = block_exclusive_scan(lane == 0 ? weq : 0, sm.wsum, tot_eq);
    int tie = ties + __shfl_sync(0xffffffffu, eq_scan, 0);
    uint32_t keepb[kPer];
    int wkeep = 0;
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const bool mine_eq = (eqb[u] >> lane) & 1u;
      const bool k_lane = ((gtb[u] >> lane) & 1u) || (mine_eq && tie + __popc(eqb[u] & lt) < take_t);
      keepb[u] = __ballot_sync(0xffffffffu, k_lane);
      tie += __popc(eqb[u]);
      wkeep += __popc(keepb[u]);
    }
    int tot_keep = 0;
    const int keep_scan = block_exclusive_scan(lane == 0 ? wkeep : 0, sm.wsum, tot_keep);
    int pos = kept + __shfl_sync(0xffffffffu, keep_scan, 0);
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      if ((keepb[u] >> lane) & 1u) {
        const int p = pos + __popc(keepb[u] & lt);
        if (p < k) out[p] = w0 + u * 32;
      }
      pos += __popc(keepb[u]);
    }
    kept += tot_keep;
    ties += tot_eq;
  }
  const int cnt = kept < k ? kept : k;
  for (int j = cnt + threadIdx.x; j < k; j += kRadixThreads) out[j] = -1;
  if (threadIdx.x == 0 && count != nullptr) count[b] = cnt;
}
}  // namespace

cudaError_t launch_cp_radix_level(const float* scores, int64_t ld, const int32_t* n_local, int B, int k, int N,
                                  int level, const int32_t* gathered, int64_t rank_stride, CpRadixState* state,
                                  int32_t* hist_out, DeviceStatus* status, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)B);
  cfg.blockDim = dim3(kRadixThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, cp_radix_level_kernel, scores, ld, n_local, k, N, level, gathered,
                                     rank_stride, state, hist_out, status);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_cp_radix_finish(const float* scores, int64_t ld, const int32_t* n_local, int B, int k, int N,
                                   int rank, const int32_t* gathered, int64_t rank_stride, const CpRadixState* state,
                                   int32_t* local_idx, int32_t* count, DeviceStatus* status, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)B);
  cfg.blockDim = dim3(kRadixThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, cp_radix_finish_kernel, scores, ld, n_local, k, N, rank, gathered,
                                     rank_stride, state, local_idx, count, status);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

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
