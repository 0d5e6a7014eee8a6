// Top-k for few long rows (decode: one row per sequence), each row spread
// over one thread-block cluster of G CTAs.  Same definition as topk.cu
// [IndexCache technical summary section 1: keep the k most relevant tokens]:
// the min(k, n) largest scores, ties to the LOWER index, ascending output,
// -1 padding.
//
// The CTAs of a row exchange everything through distributed shared memory
// and the hardware cluster barrier -- no global atomics, no spin-waits, no
// scratch to clear between calls:
//   0  each CTA loads its chunk of keys into shared memory, histograms key
//      bits [31:20] and lists its non-empty bins;
//   A  each CTA sums the G lists of its cluster into the row histogram,
//      finds the threshold bucket (the one holding the k-th largest key) and
//      the count above it, counts its own keys above the bucket and lists
//      its keys inside the bucket (the candidates);
//   B  each CTA gathers the row's candidates, finishes the radix select on
//      them (key bits [19:10], [9:0], then the index among keys equal to the
//      k-th, for the lower-index rule) -- the same answer in every CTA of
//      the row -- and writes its own chunk's selected indices, in index
//      order, at the offset given by the earlier chunks' counts.
// A CTA whose candidates overflow its shared list spills them to its slot in
// the workspace; a row with many candidates refines them in place, from the
// owners' shared memory or their slots (slow, but exact).
#include <cooperative_groups.h>

#include <atomic>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sm100.cuh"
#include "timeline.cuh"
#include "status.cuh"
#include "topk.cuh"

namespace cg = cooperative_groups;

namespace sa {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kBins1 = 4096;                // digit [31:20]
constexpr int kGroups = 8;                  // 32-key groups per warp per pass
constexpr int kPass = kThreads * kGroups;   // keys per pass (8192)
constexpr int kChunkUnit = kPass;           // chunks are whole passes
constexpr int kKeyCache = 16384;            // chunk keys kept in shared memory
constexpr int kCandLocal = 2048;            // this CTA's candidates, in shared memory
constexpr int kCandRow = 6144;              // the row's candidates gathered for the refine
constexpr int kMaxCluster = 16;
constexpr int kBitWords = 4096;             // chunks up to 131072 keys emit from a bitmap

struct Smem {
  uint32_t keys[kKeyCache];
  uint32_t hist[kBins1];
  uint2 list[kBins1];         // (bin, count) of the non-empty bins of this chunk
  uint2 cand[kCandLocal];     // (key, index) of this chunk's keys in the bucket
  uint2 row_cand[kCandRow];
  uint32_t bits[kBitWords];   // this chunk's selected keys, one bit per key
  int nlist, cnt_above, ncand, spilled;
  int cpre[kMaxCluster + 1];  // candidate prefix over the cluster's CTAs
  int peer_above[kMaxCluster], peer_spill[kMaxCluster];
  int spill_any, cand_ctr, above_ctr;
  int ws[kWarps + 1];
  int bin, before;
};

__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ int block_scan_excl(int v, int* ws, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int x = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += x;
  }
  __syncthreads();
  if (lane == 31) ws[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int w = lane < kWarps ? ws[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += x;
    }
    if (lane < kWarps) ws[lane] = wi - w;
    if (lane == kWarps - 1) ws[kWarps] = wi;
  }
  __syncthreads();
  const int ex = ws[warp] + incl - v;
  *total = ws[kWarps];
  __syncthreads();
  return ex;
}

// hist[0..nb) scanned from the top bin down: the bin where the running count
// reaches `need`; *before = count strictly above it.
__device__ void find_bin_desc(const uint32_t* hist, int nb, int need, int* ws, int* s_bin, int* s_before) {
  const int per = (nb + kThreads - 1) / kThreads;
  if (threadIdx.x == 0) {  // stays in range even if the counts fall short (a timed-out barrier)
    *s_bin = 0;
    *s_before = 0;
  }
  int local = 0;
  for (int j = 0; j < per; ++j) {
    const int bin = nb - 1 - (threadIdx.x * per + j);
    if (bin >= 0) local += (int)hist[bin];
  }
  int tot;
  int before = block_scan_excl(local, ws, &tot);
  if (before < need && need <= before + local) {
    for (int j = 0; j < per; ++j) {
      const int bin = nb - 1 - (threadIdx.x * per + j);
      if (bin < 0) break;
      const int c = (int)hist[bin];
      if (before + c >= need) {
        *s_bin = bin;
        *s_before = before;
        break;
      }
      before += c;
    }
  }
  __syncthreads();
}

// radix select, descending, over candidate values v(j) with pred(j): finds
// the need-th largest value T among those matching (prefix, mask); returns
// in *need the count of values == T that are taken, in *n_eq how many equal T.
template <class Val, class Pred>
__device__ uint32_t radix_desc(int nc, Val val, Pred pred, uint32_t prefix, uint32_t mask, const int* shifts,
                               const int* widths, int nlev, int* need, int* n_eq, Smem& sm) {
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
    find_bin_desc(sm.hist, nb, *need, sm.ws, &sm.bin, &sm.before);
    prefix |= (uint32_t)sm.bin << shift;
    mask |= (uint32_t)(nb - 1) << shift;
    *need -= sm.before;
    *n_eq = (int)sm.hist[sm.bin];
    __syncthreads();
  }
  return prefix;
}

// Pass layout: warp w covers keys [base0 + 256 w, +256) of a pass, as 8
// groups of 32 (one key per lane), so group ballots come out in index order
// and lane gi < 8 can own the word of group gi.
__device__ __forceinline__ int pass_pos(int base0, int warp, int gi, int lane) {
  return base0 + (warp * kGroups + gi) * 32 + lane;
}

__global__ void __launch_bounds__(kThreads) topk_cluster_kernel(const float* __restrict__ scores, int64_t ld,
                                                                const int32_t* __restrict__ n_valid, int n_max,
                                                                int k, int chunk, uint2* __restrict__ spill,
                                                                int32_t* __restrict__ idx,
                                                                float* __restrict__ top_scores, DeviceStatus* status) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
  cg::cluster_group cluster = cg::this_cluster();
  const int G = (int)cluster.num_blocks();
  const int c = (int)cluster.block_rank();
  const int q = blockIdx.x / G, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < kBins1; i += kThreads) sm.hist[i] = 0;
  if (tid == 0) {
    sm.cand_ctr = 0;
    sm.above_ctr = 0;
  }
  if (tid == 0) SA_TL(kTlTopk, 0);
  pdl_wait();  // the scores come from the previous kernel of the stream
  if (tid == 0) SA_TL(kTlTopk, 1);
  int n = n_valid[q];
  if (n < 0 || n > n_max) {
    if (c == 0 && tid == 0) report(status, kErrDevice, kKernTopk, q, n, n_max);
    n = n < 0 ? 0 : n_max;
  }
  const float* row = scores + (int64_t)q * ld;
  const int beg = c * chunk;
  const int len = n - beg < 0 ? 0 : (n - beg < chunk ? n - beg : chunk);
  const bool cached = chunk <= kKeyCache;
  int32_t* out = idx + (int64_t)q * k;
  float* out_s = top_scores ? top_scores + (int64_t)q * k : nullptr;
  if (n <= k) pdl_trigger();
  if (n <= k) {  // every valid key is selected (uniform over the cluster: no barrier is skipped by half of it)
    for (int i = tid; i < len; i += kThreads) {
      out[beg + i] = beg + i;
      if (out_s) out_s[beg + i] = row[beg + i];
    }
    if (c == G - 1)
      for (int p = n + tid; p < k; p += kThreads) {
        out[p] = -1;
        if (out_s) out_s[p] = 0.f;
      }
    return;
  }
  auto key_at = [&](int i) -> uint32_t { return cached ? sm.keys[i] : order_key(__ldg(&row[beg + i])); };

  // ---- phase 0: keys into shared memory, chunk histogram, non-empty bins ----
  __syncthreads();
  for (int base0 = 0; base0 < len; base0 += kPass) {
    uint32_t key[kGroups];
#pragma unroll
    for (int u = 0; u < kGroups; ++u) {  // all loads of the pass in flight together
      const int i = base0 + u * kThreads + tid;
      key[u] = i < len ? order_key(__ldg(&row[beg + i])) : 0u;
    }
#pragma unroll
    for (int u = 0; u < kGroups; ++u) {
      const int i = base0 + u * kThreads + tid;
      if (i < len) {
        if (cached) sm.keys[i] = key[u];
        atomicAdd(&sm.hist[key[u] >> 20], 1u);
      }
    }
  }
  __syncthreads();
  {
    constexpr int kPer = kBins1 / kThreads;
    int cnt = 0;
#pragma unroll
    for (int j = 0; j < kPer; ++j) cnt += sm.hist[tid * kPer + j] != 0u;
    int tot;
    int pos = block_scan_excl(cnt, sm.ws, &tot);
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const uint32_t h = sm.hist[tid * kPer + j];
      if (h) sm.list[pos++] = make_uint2((uint32_t)(tid * kPer + j), h);
    }
    if (tid == 0) sm.nlist = tot;
  }
  if (tid == 0) SA_TL(kTlTopk, 2);
  cluster.sync();
  if (tid == 0) SA_TL(kTlTopk, 3);

  // ---- phase A: row histogram, threshold bucket, this chunk's candidates ----
  for (int i = tid; i < kBins1; i += kThreads) sm.hist[i] = 0;
  __syncthreads();
  for (int r = warp; r < G; r += kWarps) {
    const Smem* peer = cluster.map_shared_rank(&sm, r);
    const int nl = peer->nlist;
    for (int e0 = 0; e0 < nl; e0 += 128) {
      uint2 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int e = e0 + u * 32 + lane;
        v[u] = e < nl ? peer->list[e] : make_uint2(0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (v[u].y) atomicAdd(&sm.hist[v[u].x & (kBins1 - 1)], v[u].y);
    }
  }
  __syncthreads();
  find_bin_desc(sm.hist, kBins1, k, sm.ws, &sm.bin, &sm.before);
  if (tid == 0) SA_TL(kTlTopk, 4);
  const int beta = sm.bin, above = sm.before;
  uint2* my_spill = spill + (int64_t)blockIdx.x * chunk;
  const bool use_bits = chunk <= kBitWords * 32;
  {
    int my_above = 0;
    for (int base0 = 0; base0 < len; base0 += kPass) {
      uint32_t key[kGroups], eqm[kGroups];
#pragma unroll
      for (int gi = 0; gi < kGroups; ++gi) {
        const int i = pass_pos(base0, warp, gi, lane);
        key[gi] = i < len ? key_at(i) : 0u;
      }
      int my = 0;
#pragma unroll
      for (int gi = 0; gi < kGroups; ++gi) {
        const bool in = pass_pos(base0, warp, gi, lane) < len;
        const int d = (int)(key[gi] >> 20);
        my_above += (in && d > beta) ? 1 : 0;
        eqm[gi] = __ballot_sync(0xffffffffu, in && d == beta);
        my += __popc(eqm[gi]);
        const uint32_t up = __ballot_sync(0xffffffffu, in && d > beta);
        if (use_bits && lane == 0) sm.bits[pass_pos(base0, warp, gi, 0) >> 5] = up;  // the group's 32 keys, one word
      }
      if (my) {  // one slot reservation per warp and pass; candidate order is free
        int slot = 0;
        if (lane == 0) slot = atomicAdd(&sm.cand_ctr, my);
        slot = __shfl_sync(0xffffffffu, slot, 0);
#pragma unroll
        for (int gi = 0; gi < kGroups; ++gi) {
          if ((eqm[gi] >> lane) & 1u) {
            const int p = slot + __popc(eqm[gi] & ((1u << lane) - 1u));
            const uint2 v = make_uint2(key[gi], (uint32_t)(beg + pass_pos(base0, warp, gi, lane)));
            if (p < kCandLocal) sm.cand[p] = v;
            else my_spill[p] = v;
          }
          slot += __popc(eqm[gi]);
        }
      }
    }
    // this chunk's count above the bucket: warp sums, one shared atomic each
    const int wsum = __reduce_add_sync(0xffffffffu, my_above);
    if (lane == 0 && wsum) atomicAdd(&sm.above_ctr, wsum);
    __syncthreads();
    const int ncand = sm.cand_ctr;
    const int spilled = ncand > kCandLocal;
    if (spilled)  // the whole list then lives in the workspace
      for (int p = tid; p < kCandLocal; p += kThreads) my_spill[p] = sm.cand[p];
    // push this chunk's counts into every CTA of the row (read after the barrier)
    if (tid < G) {
      Smem* peer = cluster.map_shared_rank(&sm, tid);
      peer->cpre[c + 1] = ncand;
      peer->peer_above[c] = sm.above_ctr;
      peer->peer_spill[c] = spilled;
    }
  }
  if (tid == 0) SA_TL(kTlTopk, 5);
  cluster.sync();
  if (tid == 0) SA_TL(kTlTopk, 6);

  // ---- phase B: exact k-th key, then this chunk's part of the output ----
  if (warp == 0) {  // candidate prefix over the chunks, keys above the bucket before this chunk
    const int n_r = lane < G ? sm.cpre[lane + 1] : 0;
    int incl = n_r;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += x;
    }
    const int ab = __reduce_add_sync(0xffffffffu, lane < c ? sm.peer_above[lane] : 0);
    const int sp = __reduce_or_sync(0xffffffffu, lane < G ? sm.peer_spill[lane] : 0);
    __syncwarp();
    if (lane < G) sm.cpre[lane + 1] = incl;
    if (lane == 0) {
      sm.cpre[0] = 0;
      sm.before = ab;
      sm.spill_any = sp;
    }
  }
  __syncthreads();
  const int above_before = sm.before;
  const int nc = sm.cpre[G];
  const bool fast = !sm.spill_any && nc <= kCandRow;
  auto cand_at = [&](int j) -> uint2 {  // j-th candidate of the row, from its owner
    int lo = 0, hi = G;                 // owner r with cpre[r] <= j < cpre[r + 1]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (sm.cpre[mid] <= j) lo = mid; else hi = mid;
    }
    const int e = j - sm.cpre[lo];
    if (sm.peer_spill[lo]) return __ldcg(&spill[((int64_t)q * G + lo) * chunk + e]);
    return cluster.map_shared_rank(&sm, lo)->cand[e];
  };
  if (fast) {
    for (int j0 = 0; j0 < nc; j0 += 4 * kThreads) {
      uint2 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = j0 + u * kThreads + tid;
        v[u] = j < nc ? cand_at(j) : make_uint2(0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = j0 + u * kThreads + tid;
        if (j < nc) sm.row_cand[j] = v[u];
      }
    }
    __syncthreads();
  }
  if (tid == 0) SA_TL(kTlTopk, 7);
  auto ckey = [&](int j) { return fast ? sm.row_cand[j].x : cand_at(j).x; };
  auto cidx = [&](int j) { return fast ? sm.row_cand[j].y : cand_at(j).y; };
  int need = k - above, n_eq = 0;
  const int ks[2] = {10, 0}, kw[2] = {10, 10};
  const uint32_t T = radix_desc(nc, ckey, [](int) { return true; }, (uint32_t)beta << 20, 0xFFF00000u, ks, kw, 2,
                                &need, &n_eq, sm);
  if (tid == 0) SA_TL(kTlTopk, 8);
  uint32_t cut = 0xFFFFFFFFu;
  if (need < n_eq) {
    // the `need` lowest indices among keys == T: largest values of ~index
    int need2 = need, n2 = 0;
    const int is[3] = {21, 10, 0}, iw[3] = {11, 11, 10};
    const uint32_t V = radix_desc(nc, [&](int j) { return ~cidx(j); }, [&](int j) { return ckey(j) == T; }, 0u, 0u,
                                  is, iw, 3, &need2, &n2, sm);
    cut = ~V;
  }
  // selected candidates of earlier chunks (candidates are grouped by owner,
  // owners in chunk order)
  int sel_before = 0;
  for (int j = tid; j < sm.cpre[c]; j += kThreads) {
    const uint32_t kx = ckey(j), ix = cidx(j);
    if (kx > T || (kx == T && ix <= cut)) ++sel_before;
  }
  int tot_sel_before;
  block_scan_excl(sel_before, sm.ws, &tot_sel_before);
  int written = above_before + tot_sel_before;
  if (tid == 0) SA_TL(kTlTopk, 9);
  // The next kernel of the stream may start launching now, a few us before
  // this one ends, so its set-up overlaps the emission below.  Letting it
  // launch at entry put its waiting CTAs on the free SMs for the whole
  // top-k, which measured 4 us slower inside the decode step (18.0 against
  // 13.8 us).
  pdl_trigger();
  // this CTA reads nothing of its peers from here on; the matching wait
  // before exit keeps its own lists alive until every peer is past this point
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  if (use_bits) {
    // the keys above the bucket are already set; add this chunk's kept bucket
    // keys, then emit the set bits in index order
    const int my_nc = sm.cand_ctr;
    const bool mine_spilled = my_nc > kCandLocal;
    for (int j = tid; j < my_nc; j += kThreads) {
      const uint2 v = mine_spilled ? __ldcg(&my_spill[j]) : sm.cand[j];
      if (v.x > T || (v.x == T && v.y <= cut)) {
        const uint32_t li = v.y - (uint32_t)beg;
        atomicOr(&sm.bits[li >> 5], 1u << (li & 31));
      }
    }
    __syncthreads();
    const int nwl = (len + 31) >> 5;
    const int per = (nwl + kThreads - 1) / kThreads;
    int cnt = 0;
    for (int q2 = 0; q2 < per; ++q2) {
      const int wi = tid * per + q2;
      if (wi < nwl) cnt += __popc(sm.bits[wi]);
    }
    int tot;
    int pos = written + block_scan_excl(cnt, sm.ws, &tot);
    for (int q2 = 0; q2 < per; ++q2) {
      const int wi = tid * per + q2;
      if (wi >= nwl) break;
      uint32_t x = sm.bits[wi];
      while (x) {
        const int b = __ffs(x) - 1;
        x &= x - 1;
        const int i = beg + (wi << 5) + b;
        if (pos < k) {
          out[pos] = i;
          if (out_s) out_s[pos] = row[i];
        }
        ++pos;
      }
    }
    if (tid == 0) SA_TL(kTlTopk, 10);
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
    if (tid == 0) SA_TL(kTlTopk, 11);
    return;
  }
  for (int base0 = 0; base0 < len; base0 += kPass) {
    uint32_t key[kGroups];
#pragma unroll
    for (int gi = 0; gi < kGroups; ++gi) {
      const int i = pass_pos(base0, warp, gi, lane);
      key[gi] = i < len ? key_at(i) : 0u;
    }
    uint32_t x = 0;
#pragma unroll
    for (int gi = 0; gi < kGroups; ++gi) {
      const int i = pass_pos(base0, warp, gi, lane);
      const int d = (int)(key[gi] >> 20);
      const bool sel = i < len && (d > beta || (d == beta && (key[gi] > T || (key[gi] == T && (uint32_t)(beg + i) <= cut))));
      const uint32_t w = __ballot_sync(0xffffffffu, sel);
      if (lane == gi) x = w;
    }
    int tot;
    int pos = written + block_scan_excl(__popc(x), sm.ws, &tot);
    const int base = beg + pass_pos(base0, warp, lane, 0);  // lane < 8: its group's first key
    while (x) {
      const int b = __ffs(x) - 1;
      x &= x - 1;
      if (pos < k) {
        out[pos] = base + b;
        if (out_s) out_s[pos] = row[base + b];
      }
      ++pos;
    }
    written += tot;
  }
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

struct Plan {
  int G, chunk;
};

// G: CTAs per row (a cluster), a power of two up to max_g with Nq * G <= SMs
Plan plan_for(int Nq, int n_max, int num_sms, int max_g) {
  Plan p;
  int G = 1;
  while (G * 2 <= max_g && (int64_t)Nq * G * 2 <= num_sms && (int64_t)G * kChunkUnit < n_max) G *= 2;
  int64_t chunk = ((int64_t)n_max + G - 1) / G;
  chunk = (chunk + kChunkUnit - 1) / kChunkUnit * kChunkUnit;
  p.G = G;
  p.chunk = (int)chunk;
  return p;
}

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

// Largest cluster the device schedules for this kernel (16 needs the
// non-portable size; some parts only give 8).  Looked up once per device.
int max_cluster() {
  static std::atomic<int> cached[64];  // per device; every writer stores the same value
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 8;
  if (const int c = cached[dev].load(std::memory_order_relaxed)) return c;
  int g = 8;
  if (cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess &&
      ensure_smem(topk_cluster_kernel, sizeof(Smem)) == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kMaxCluster);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = sizeof(Smem);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kMaxCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, topk_cluster_kernel, &cfg) == cudaSuccess && n >= 1) g = kMaxCluster;
  }
  cudaGetLastError();
  cached[dev].store(g, std::memory_order_relaxed);
  return g;
}

}  // namespace

size_t topk_split_ws_bytes(int Nq, int n_max, int num_sms) {
  // candidate spill slots: one chunk per CTA, for either cluster size
  size_t most = 0;
  for (int g = 8; g <= kMaxCluster; g *= 2) {
    const Plan p = plan_for(Nq, n_max, num_sms, g);
    const size_t b = 8ull * p.chunk * (size_t)Nq * p.G;
    if (b > most) most = b;
  }
  return round256(most);
}

bool topk_use_split(int Nq, int n_max, int num_sms) { return Nq > 0 && Nq * 2 <= num_sms && n_max > 8192; }

cudaError_t launch_topk_split(const float* scores, int64_t ld, const int32_t* n_valid, int Nq, int n_max, int k,
                              int32_t* idx, float* top_scores, DeviceStatus* status, void* scratch, int num_sms,
                              cudaStream_t stream) {
  const Plan p = plan_for(Nq, n_max, num_sms, max_cluster());
  cudaError_t e = ensure_smem(topk_cluster_kernel, sizeof(Smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(Nq * p.G));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = sizeof(Smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;  // the CTAs of one row form one cluster
  attr[0].val.clusterDim.x = p.G;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1] = pdl_attribute();
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, topk_cluster_kernel, scores, ld, n_valid, n_max, k, p.chunk,
                         reinterpret_cast<uint2*>(scratch), idx, top_scores, status);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace sa

SA_TL_SETTER(sa_timeline_set_topk)
