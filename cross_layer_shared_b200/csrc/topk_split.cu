// Top-k for few long rows (decode: one row per sequence), spread over many
// CTAs per row.  Same definition as topk.cu [IndexCache technical summary
// section 1: keep the k most relevant tokens]: the min(k, n) largest scores,
// ties to the lower index, ascending output, -1 padding.
//
// Two kernels, no spin-wait anywhere (the last CTA of a row to finish does
// the row's serial part; it learns it is last from an atomic ticket):
//   hist    each CTA histograms key bits [31:20] of its chunk in shared
//           memory and adds it into the row's global histogram; the row's
//           last CTA finds the threshold bucket and how many keys lie above.
//   select  each CTA turns its chunk into bitmap words (warp ballot: key
//           above the bucket = selected) and appends the keys inside the
//           bucket to the row's candidate list; the row's last CTA finishes
//           the radix select on the candidates (key bits [19:10], [9:0], then
//           the index among keys equal to the k-th, for the lower-index
//           rule), ORs the winners into the bitmap and emits the set bits in
//           index order from a block-wide prefix sum of popcounts.
#include <cuda_runtime.h>
#include <stdint.h>

#include "sm100.cuh"
#include "status.cuh"
#include "topk.cuh"

namespace sa {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBins1 = 4096;

struct RowState {
  int beta;    // threshold bucket of bits [31:20]; -1: the whole row is selected
  int above;   // keys in buckets above beta
  int n;       // valid length
  int ncand;   // keys appended to the candidate list
  int ticket1;
  int ticket2;
  int pad[2];
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

__global__ void __launch_bounds__(kThreads) topk_hist_kernel(const float* __restrict__ scores, int64_t ld,
                                                             const int32_t* __restrict__ n_valid, int n_max, int k,
                                                             int chunk, uint32_t* __restrict__ hist,
                                                             RowState* __restrict__ st, DeviceStatus* status) {
  __shared__ uint32_t sh[kBins1];
  __shared__ int ws[kWarps + 1];
  __shared__ int s_last, s_bin, s_before;
  const int q = blockIdx.y, c = blockIdx.x, tid = threadIdx.x;
  int n = n_valid[q];
  if (n < 0 || n > n_max) {
    if (c == 0 && tid == 0) report(status, kErrDevice, kKernTopk, q, n, n_max);
    n = n < 0 ? 0 : n_max;
  }
  const float* row = scores + (int64_t)q * ld;
  for (int i = tid; i < kBins1; i += kThreads) sh[i] = 0;
  __syncthreads();
  const int beg = c * chunk, end = min(n, beg + chunk);
  if (n > k)
    for (int i = beg + tid; i < end; i += kThreads) atomicAdd(&sh[order_key(row[i]) >> 20], 1u);
  __syncthreads();
  uint32_t* h = hist + (int64_t)q * kBins1;
  if (n > k)
    for (int i = tid; i < kBins1; i += kThreads)
      if (sh[i]) atomicAdd(&h[i], sh[i]);
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(&st[q].ticket1, 1) == (int)gridDim.x - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (n <= k) {
    if (tid == 0) {
      st[q].beta = -1;
      st[q].above = n;
      st[q].n = n;
    }
    return;
  }
  for (int i = tid; i < kBins1; i += kThreads) sh[i] = __ldcg(&h[i]);
  __syncthreads();
  find_bin_desc(sh, kBins1, k, ws, &s_bin, &s_before);
  if (tid == 0) {
    st[q].beta = s_bin;
    st[q].above = s_before;
    st[q].n = n;
  }
}

// radix select, descending, over candidate values v(j) with pred(j): finds
// the need-th largest value T among those matching (prefix, mask); returns
// in *need the count of values == T that are taken, in *n_eq how many equal T.
template <class Val, class Pred>
__device__ uint32_t radix_desc(int nc, Val val, Pred pred, uint32_t prefix, uint32_t mask, const int* shifts,
                               const int* widths, int nlev, int* need, int* n_eq, uint32_t* sh, int* ws, int* s_bin,
                               int* s_before) {
  for (int lv = 0; lv < nlev; ++lv) {
    const int shift = shifts[lv], nb = 1 << widths[lv];
    for (int i = threadIdx.x; i < nb; i += kThreads) sh[i] = 0;
    __syncthreads();
    for (int j = threadIdx.x; j < nc; j += kThreads) {
      if (!pred(j)) continue;
      const uint32_t v = val(j);
      if ((v & mask) == prefix) atomicAdd(&sh[(v >> shift) & (uint32_t)(nb - 1)], 1u);
    }
    __syncthreads();
    find_bin_desc(sh, nb, *need, ws, s_bin, s_before);
    prefix |= (uint32_t)*s_bin << shift;
    mask |= (uint32_t)(nb - 1) << shift;
    *need -= *s_before;
    *n_eq = (int)sh[*s_bin];
    __syncthreads();
  }
  return prefix;
}

constexpr int kGroups = 8;            // 32-key groups per warp per chunk pass (registers)
constexpr int kCandSmem = 6144;       // candidates refined in shared memory
constexpr int kWordsSmem = 4096;      // bitmap words staged in shared memory (rows <= 131072)

struct SelectSmem {
  uint2 cand[kCandSmem];
  uint32_t words[kWordsSmem];
  uint32_t hist[2048];
  int ws[kWarps + 1];
  int warp_cnt[kWarps];
  int cta_base;
  int last, bin, before;
};

__global__ void __launch_bounds__(kThreads) topk_select_kernel(const float* __restrict__ scores, int64_t ld, int k,
                                                               int chunk, RowState* __restrict__ st,
                                                               uint32_t* __restrict__ bitmap, int wpr,
                                                               uint2* __restrict__ cand, int cap,
                                                               int32_t* __restrict__ idx, float* __restrict__ top_scores) {
  extern __shared__ uint8_t smem_raw[];
  SelectSmem& sm = *reinterpret_cast<SelectSmem*>(smem_raw);
  const int q = blockIdx.y, c = blockIdx.x, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int beta = __ldcg(&st[q].beta), above = __ldcg(&st[q].above), n = __ldcg(&st[q].n);
  const float* row = scores + (int64_t)q * ld;
  uint32_t* bm = bitmap + (int64_t)q * wpr;
  uint2* cq = cand + (int64_t)q * cap;

  // ---- this CTA's chunk: selected-bit words and threshold-bucket candidates ----
  const int beg = c * chunk, end = min(n, beg + chunk);
  for (int base0 = beg; base0 < end; base0 += kThreads * kGroups) {
    uint32_t key[kGroups];
    uint32_t eqm[kGroups];
    int my = 0;  // candidates of this warp in this pass
#pragma unroll
    for (int gi = 0; gi < kGroups; ++gi) {
      const int base = base0 + (gi * kWarps + warp) * 32;
      const int i = base + lane;
      const bool in = i < end;
      key[gi] = in ? order_key(row[i]) : 0u;
      const int d = (int)(key[gi] >> 20);
      const bool sel = in && (beta < 0 || d > beta);
      const bool eq = in && beta >= 0 && d == beta;
      const uint32_t word = __ballot_sync(0xffffffffu, sel);
      if (lane == 0 && base < end) bm[base >> 5] = word;
      eqm[gi] = __ballot_sync(0xffffffffu, eq);
      my += __popc(eqm[gi]);
    }
    if (lane == 0) sm.warp_cnt[warp] = my;
    __syncthreads();
    if (tid == 0) {
      int tot = 0;
      for (int w = 0; w < kWarps; ++w) {
        const int x = sm.warp_cnt[w];
        sm.warp_cnt[w] = tot;
        tot += x;
      }
      sm.cta_base = tot ? atomicAdd(&st[q].ncand, tot) : 0;  // one reservation per CTA
    }
    __syncthreads();
    int pos = sm.cta_base + sm.warp_cnt[warp];
#pragma unroll
    for (int gi = 0; gi < kGroups; ++gi) {
      const int base = base0 + (gi * kWarps + warp) * 32;
      if ((eqm[gi] >> lane) & 1u) {
        const int p = pos + __popc(eqm[gi] & ((1u << lane) - 1u));
        if (p < cap) cq[p] = make_uint2(key[gi], (uint32_t)(base + lane));
      }
      pos += __popc(eqm[gi]);
    }
    __syncthreads();
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) sm.last = atomicAdd(&st[q].ticket2, 1) == (int)gridDim.x - 1;
  __syncthreads();
  if (!sm.last) return;
  __threadfence();

  // ---- the row's last CTA ---------------------------------------------------
  const int nw = (n + 31) >> 5;
  const bool words_in_smem = nw <= kWordsSmem;
  if (words_in_smem)
    for (int w = tid; w < nw; w += kThreads) sm.words[w] = __ldcg(&bm[w]);
  if (beta >= 0) {
    int nc = __ldcg(&st[q].ncand);
    nc = nc < cap ? nc : cap;
    const bool in_smem = nc <= kCandSmem;
    if (in_smem)
      for (int j = tid; j < nc; j += kThreads) sm.cand[j] = __ldcg(&cq[j]);
    __syncthreads();
    const uint2* cs = in_smem ? sm.cand : cq;
    auto ckey = [&](int j) { return in_smem ? sm.cand[j].x : __ldcg(&cq[j].x); };
    auto cidx = [&](int j) { return in_smem ? sm.cand[j].y : __ldcg(&cq[j].y); };
    int need = k - above;
    int n_eq = 0;
    const int ks[2] = {10, 0}, kw[2] = {10, 10};
    const uint32_t T = radix_desc(nc, ckey, [](int) { return true; }, (uint32_t)beta << 20, 0xFFF00000u, ks, kw,
                                  2, &need, &n_eq, sm.hist, sm.ws, &sm.bin, &sm.before);
    uint32_t cut = 0xFFFFFFFFu;
    if (need < n_eq) {
      // the `need` lowest indices among keys == T: largest values of ~index
      int need2 = need, n2 = 0;
      const int is[3] = {21, 10, 0}, iw[3] = {11, 11, 10};
      const uint32_t V = radix_desc(nc, [&](int j) { return ~cidx(j); }, [&](int j) { return ckey(j) == T; }, 0u,
                                    0u, is, iw, 3, &need2, &n2, sm.hist, sm.ws, &sm.bin, &sm.before);
      cut = ~V;
    }
    (void)cs;
    for (int j = tid; j < nc; j += kThreads) {
      const uint32_t kx = ckey(j), ix = cidx(j);
      if (kx > T || (kx == T && ix <= cut)) {
        if (words_in_smem) atomicOr(&sm.words[ix >> 5], 1u << (ix & 31));
        else atomicOr(&bm[ix >> 5], 1u << (ix & 31));
      }
    }
    if (!words_in_smem) __threadfence();
  }
  __syncthreads();

  // ---- emit set bits in index order ----------------------------------------
  int32_t* out = idx + (int64_t)q * k;
  float* out_s = top_scores ? top_scores + (int64_t)q * k : nullptr;
  constexpr int kWpt = 8;
  int written = 0;
  for (int w0 = 0; w0 < nw; w0 += kThreads * kWpt) {
    uint32_t wv[kWpt];
    int cnt = 0;
#pragma unroll
    for (int j = 0; j < kWpt; ++j) {
      const int wi = w0 + tid * kWpt + j;
      wv[j] = wi < nw ? (words_in_smem ? sm.words[wi] : __ldcg(&bm[wi])) : 0u;
      if (wi == nw - 1 && (n & 31)) wv[j] &= (1u << (n & 31)) - 1u;
      cnt += __popc(wv[j]);
    }
    int tot;
    int pos = written + block_scan_excl(cnt, sm.ws, &tot);
#pragma unroll
    for (int j = 0; j < kWpt; ++j) {
      uint32_t x = wv[j];
      const int wi = w0 + tid * kWpt + j;
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
    written += tot;
  }
  for (int p = written + tid; p < k; p += kThreads) {
    out[p] = -1;
    if (out_s) out_s[p] = 0.f;
  }
}

int chunk_for(int Nq, int n_max, int num_sms) {
  // about one CTA per SM over all rows; a multiple of one select pass
  int64_t want = ((int64_t)Nq * n_max + num_sms - 1) / num_sms;
  const int pass = kThreads * kGroups;
  want = (want + pass - 1) / pass * pass;
  if (want < pass) want = pass;
  return (int)want;
}

}  // namespace

size_t topk_split_ws_bytes(int Nq, int n_max) {
  const size_t wpr = ((size_t)n_max + 31) / 32;
  auto r = [](size_t x) { return (x + 255) / 256 * 256; };
  return r(sizeof(RowState) * Nq) + r(4ull * kBins1 * Nq) + r(4 * wpr * Nq) + r(8ull * (size_t)n_max * Nq);
}

bool topk_use_split(int Nq, int n_max, int num_sms) { return Nq > 0 && Nq * 2 <= num_sms && n_max > 8192; }

cudaError_t launch_topk_split(const float* scores, int64_t ld, const int32_t* n_valid, int Nq, int n_max, int k,
                              int32_t* idx, float* top_scores, DeviceStatus* status, void* scratch, int num_sms,
                              cudaStream_t stream) {
  const size_t wpr = ((size_t)n_max + 31) / 32;
  auto r = [](size_t x) { return (x + 255) / 256 * 256; };
  uint8_t* p = reinterpret_cast<uint8_t*>(scratch);
  RowState* st = reinterpret_cast<RowState*>(p);
  uint32_t* hist = reinterpret_cast<uint32_t*>(p + r(sizeof(RowState) * Nq));
  uint32_t* bm = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(hist) + r(4ull * kBins1 * Nq));
  uint2* cand = reinterpret_cast<uint2*>(reinterpret_cast<uint8_t*>(bm) + r(4 * wpr * Nq));
  // row states and histograms start at zero every call
  cudaError_t e = cudaMemsetAsync(p, 0, r(sizeof(RowState) * Nq) + r(4ull * kBins1 * Nq), stream);
  if (e != cudaSuccess) return e;
  const int chunk = chunk_for(Nq, n_max, num_sms);
  const dim3 grid((n_max + chunk - 1) / chunk, Nq);
  topk_hist_kernel<<<grid, kThreads, 0, stream>>>(scores, ld, n_valid, n_max, k, chunk, hist, st, status);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = ensure_smem(topk_select_kernel, sizeof(SelectSmem));
  if (e != cudaSuccess) return e;
  topk_select_kernel<<<grid, kThreads, sizeof(SelectSmem), stream>>>(scores, ld, k, chunk, st, bm, (int)wpr, cand,
                                                                     n_max, idx, top_scores);
  return cudaGetLastError();
}

}  // namespace sa
