// Indexer-layer attention for the CLSA routing reading: dense decode
// attention of one layer over every cached token, and the routing score of
// each token, the sum over query heads of its attention weight.
//
// [CLSA news article "Le routage partage entre couches accelere l'attention
//  sparse de 7x sans perte de qualite", section "La precision reste stable":
//  the routing index is computed once from the attention scores of the
//  indexer layer, which sees the same query state and cache as every other
//  layer.]
//   z[h,t] = scale * (Q[b,h] . K[g(h),t]),  p[h,t] = softmax_t z[h,t]
//   O[b,h] = sum_t p[h,t] V[g(h),t],        route[b,t] = sum_h p[h,t]
//
// HBM-bound on CUDA cores.  A (sequence, KV head) has G = Hq/Hkv query rows
// (4 or 8 here), so every 256-byte K or V row feeds G dot products of
// length 128: 4-8 flop per byte, a GEMV below the fp32 ridge.  A 128-row
// tensor-core tile would be 94-97 % padding.
//
// Partial kernel: one CTA per (2048-key chunk, KV head, sequence).
//   Warp 8 streams the chunk's K rows, then its V rows, in 32-row tiles
//   (8 KB, contiguous: cp.async.bulk) through a 4-stage ring.
//   Warps 0-7, phase 1: the logits of the chunk, in log2 units, into shared
//   memory (thread = one key x 16 of its 128 dims, then an 8-lane sum).
//   Then per head (warp h): the chunk max m, p = 2^(z - m) in place,
//   l = sum p, and z out to global memory for the routing scores.
//   Phase 2: o[h] = sum_t p[h,t] V[t] (thread = 4 dims x 2 heads x one
//   residue class of rows; the row classes are summed at the end).
//   Writes (m, l) and o per (head, chunk).
// Combine kernel: per sequence, CTAs 0..n_tc-1 write the routing scores of
//   1024 tokens each, r_t = sum_h 2^(z[h,t] - M_h) / L_h, with (M_h, L_h) the
//   sequence-wide max and sum merged from the partials; CTA n_tc + g merges
//   the dense output of KV head g's query heads.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "route_attn.cuh"
#include "sm100.cuh"

namespace sa {
namespace {

constexpr int kD = 128;
constexpr int kRows = 32;  // key rows per ring tile
constexpr int kStages = 4;
constexpr int kCompWarps = 8;
constexpr int kPartThreads = 32 * (kCompWarps + 1);
constexpr int kTileBytes = kRows * kD * 2;
constexpr int kTokPerRouteCta = 1024;

template <int G>
struct PartLayout {
  static constexpr int kRingOff = 0;                             // [kStages][kRows][128] bf16
  static constexpr int kZOff = kRingOff + kStages * kTileBytes;  // [G][kRouteChunk] fp32: z, then p
  static constexpr int kQOff = kZOff + G * kRouteChunk * 4;      // [G][4][8][4] fp32 (see q_slot)
  static constexpr int kBarOff = kQOff + G * kD * 4;             // full[kStages] empty[kStages]
  static constexpr int kFlagOff = kBarOff + 16 * kStages;
  static constexpr size_t kSmem = kFlagOff + 16;
  static_assert(kSmem <= 232448, "shared memory budget");
};

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void comp_bar() { asm volatile("bar.sync 1, %0;" ::"n"(32 * kCompWarps) : "memory"); }

// lane 0 waits, the verdict is the warp's
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, kWaitLimitNs);
  return __shfl_sync(0xffffffffu, ok, 0);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Slot of query dim c of head h in shared memory: the 16 dims a phase-1
// thread dq uses (8dq..8dq+7, 64+8dq..64+8dq+7) are four float4 whose j-th
// ones sit side by side for dq = 0..7, so eight lanes read 128 contiguous bytes.
__device__ __forceinline__ int q_slot(int h, int c) {
  const int dq = (c & 63) >> 3;
  const int e = ((c >> 6) << 3) | (c & 7);  // 0..15 within the thread's dims
  return ((h * 4 + (e >> 2)) * 8 + dq) * 4 + (e & 3);
}

// a shared-memory load the compiler keeps in the loop (hoisting the query
// slices out of it would hold 16*G registers and cost a resident CTA)
__device__ __forceinline__ float4 lds_f4(const float* p) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(smem_u32(p)));
  return v;
}

__device__ __forceinline__ void unpack8(const uint4 u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

// Valid length of sequence b, or 0 (reported once) when its rows would fall
// outside the cache.
__device__ __forceinline__ int checked_len(const RouteArgs& a, int b, bool report_it) {
  const int len = a.seq_len[b];
  const int64_t off = a.seq_off[b];
  if (len < 0 || len > a.S_max || off < 0 || off + len > a.n_tokens) {
    if (report_it) report(a.status, kErrDevice, kKernRoute, b, len, a.S_max);
    return 0;
  }
  return len;
}

template <int G>
__global__ void __launch_bounds__(kPartThreads, 3) indexer_layer_partial_kernel(const RouteArgs a) {
  using Lay = PartLayout<G>;
  extern __shared__ __align__(128) uint8_t smem[];
  uint16_t* ring = reinterpret_cast<uint16_t*>(smem + Lay::kRingOff);
  float* zs = reinterpret_cast<float*>(smem + Lay::kZOff);
  float* qs = reinterpret_cast<float*>(smem + Lay::kQOff);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Lay::kBarOff);
  uint64_t* empty = full + kStages;
  int* abort_flag = reinterpret_cast<int*>(smem + Lay::kFlagOff);

  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_trigger();
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kCompWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  // everything below reads what earlier kernels of the stream wrote
  pdl_wait();
  const int len = checked_len(a, b, split == 0 && g == 0 && tid == 0);
  const int t0 = split * kRouteChunk;
  const int n = max(0, min(kRouteChunk, len - t0));  // keys of this chunk
  const int nt = (n + kRows - 1) / kRows;             // K tiles, then as many V tiles
  const int64_t row0 = a.seq_off[b] * a.Hkv + (int64_t)g * len + t0;
  const int h0 = g * G;
  for (int e = tid; e < G * kD; e += kPartThreads) {
    const uint32_t q16 = a.Q[((int64_t)b * a.Hq + h0) * kD + e];
    qs[q_slot(e / kD, e % kD)] = __uint_as_float(q16 << 16);
  }
  __syncthreads();

  if (warp == kCompWarps) {
    // ---------------- producer: K tiles, then V tiles ----------------
    if (lane == 0) {
      int i = 0;
      for (; i < 2 * nt; ++i) {
        const int s = i % kStages;
        if (!mbar_wait(&empty[s], ((i / kStages) & 1) ^ 1, kWaitLimitNs)) {
          report(a.status, kErrTimeout, kKernRoute, b, split, i);
          break;
        }
        const int tile = i < nt ? i : i - nt;
        const uint32_t bytes = (uint32_t)min(kRows, n - tile * kRows) * kD * 2;
        const uint16_t* src = (i < nt ? a.K : a.V) + (row0 + (int64_t)tile * kRows) * kD;
        mbar_arrive_expect_tx(&full[s], bytes);
        bulk_load(ring + s * kRows * kD, src, bytes, &full[s]);
      }
      // every copy issued lands before the CTA exits
      for (int j = max(0, i - kStages); j < i; ++j) mbar_wait(&full[j % kStages], (j / kStages) & 1, kWaitLimitNs);
    }
    return;
  }

  // ---------------- phase 1: logits of the chunk ----------------
  // thread: key row kr of the tile, dims [8dq, 8dq+8) and [64+8dq, 64+8dq+8)
  // (eight lanes of a row read 128 contiguous bytes: no bank conflict)
  const int kr = warp * 4 + (lane >> 3);
  const int dq = lane & 7;
  for (int j = 0; j < nt; ++j) {
    const int s = j % kStages;
    if (!warp_wait(&full[s], (j / kStages) & 1)) {
      if (lane == 0) {
        report(a.status, kErrTimeout, kKernRoute, b, split, 1000000 + j);
        atomicExch(abort_flag, 1);
      }
      break;
    }
    const uint16_t* kt = ring + s * kRows * kD + kr * kD;
    float kf[16];
    unpack8(*reinterpret_cast<const uint4*>(kt + 8 * dq), kf);
    unpack8(*reinterpret_cast<const uint4*>(kt + 64 + 8 * dq), kf + 8);
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    float acc[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float x = 0.f;
#pragma unroll
      for (int j4 = 0; j4 < 4; ++j4) {
        const float4 q4 = lds_f4(qs + ((h * 4 + j4) * 8 + dq) * 4);
        x = fmaf(q4.x, kf[4 * j4], x);
        x = fmaf(q4.y, kf[4 * j4 + 1], x);
        x = fmaf(q4.z, kf[4 * j4 + 2], x);
        x = fmaf(q4.w, kf[4 * j4 + 3], x);
      }
      acc[h] = x;
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
#pragma unroll
      for (int o = 4; o > 0; o >>= 1) acc[h] += __shfl_xor_sync(0xffffffffu, acc[h], o);
    }
    const int t = j * kRows + kr;
    if (dq == 0 && t < n) {
#pragma unroll
      for (int h = 0; h < G; ++h) zs[h * kRouteChunk + t] = acc[h] * a.scale_log2;
    }
  }
  comp_bar();
  const bool aborted = *reinterpret_cast<volatile int*>(abort_flag) != 0;
  if (aborted) return;

  // ---------------- per head: chunk max, weights in place, sum ----------------
  if (warp < G) {
    float* zr = zs + warp * kRouteChunk;
    float m = -INFINITY;
    for (int t = lane; t < n; t += 32) m = fmaxf(m, zr[t]);
    m = warp_max(m);
    float* zg = a.z + ((int64_t)b * a.Hq + h0 + warp) * a.zld + t0;
    float l = 0.f;
    for (int t = lane; t < n; t += 32) {
      const float z = zr[t];
      zg[t] = z;
      const float p = exp2f(z - m);
      zr[t] = p;
      l += p;
    }
    l = warp_sum(l);
    if (lane == 0) a.part_ml[((int64_t)b * a.Hq + h0 + warp) * a.n_split + split] = make_float2(m, l);
  }
  comp_bar();

  // ---------------- phase 2: o[h] = sum_t p[h,t] V[t] ----------------
  // thread: dims [4 dq4, 4 dq4 + 4) of HP heads, rows r = rg (mod NRG) of
  // each tile; the NRG row groups are summed through shared memory at the end
  constexpr int HP = G < 2 ? G : 2;         // heads per thread
  constexpr int NHS = G / HP;               // head slots
  constexpr int NRG = kCompWarps / NHS;     // row groups (8, 8, 4, 2 for G = 1, 2, 4, 8)
  const int dq4 = tid & 31;
  const int hs = (tid >> 5) % NHS;
  const int rg = (tid >> 5) / NHS;
  float o[HP][4];
#pragma unroll
  for (int x = 0; x < HP; ++x)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[x][e] = 0.f;
  bool ok = true;
  for (int j = 0; j < nt; ++j) {
    const int i = nt + j, s = i % kStages;
    if (!warp_wait(&full[s], (i / kStages) & 1)) {
      if (lane == 0) report(a.status, kErrTimeout, kKernRoute, b, split, 2000000 + j);
      ok = false;
      break;
    }
    const int rows = min(kRows, n - j * kRows);
    const uint2* vt = reinterpret_cast<const uint2*>(ring + s * kRows * kD) + dq4;
    const float* pr = zs + (hs * HP) * kRouteChunk + j * kRows;
#pragma unroll 4
    for (int r = rg; r < rows; r += NRG) {
      const uint2 v4 = vt[r * (kD / 4)];
      const float v[4] = {__uint_as_float(v4.x << 16), __uint_as_float(v4.x & 0xffff0000u),
                          __uint_as_float(v4.y << 16), __uint_as_float(v4.y & 0xffff0000u)};
#pragma unroll
      for (int x = 0; x < HP; ++x) {
        const float p = pr[x * kRouteChunk + r];
#pragma unroll
        for (int e = 0; e < 4; ++e) o[x][e] = fmaf(p, v[e], o[x][e]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
  if (!ok && lane == 0) atomicExch(abort_flag, 1);
  // sum the row groups (the weights are no longer needed: reuse their space);
  // every compute warp reaches each barrier, a warp that gave up included
  comp_bar();
  if (*reinterpret_cast<volatile int*>(abort_flag) != 0) return;
  float* red = zs;  // [NRG][G][128]
#pragma unroll
  for (int x = 0; x < HP; ++x)
    *reinterpret_cast<float4*>(red + ((rg * G) + hs * HP + x) * kD + 4 * dq4) =
        make_float4(o[x][0], o[x][1], o[x][2], o[x][3]);
  comp_bar();
  for (int e = tid; e < G * kD; e += 32 * kCompWarps) {
    float sum = 0.f;
#pragma unroll
    for (int q = 0; q < NRG; ++q) sum += red[q * G * kD + e];
    a.part_o[(((int64_t)b * a.Hq + h0 + e / kD) * a.n_split + split) * kD + e % kD] = sum;
  }
}

template <int G>
__global__ void __launch_bounds__(256) indexer_layer_combine_kernel(const RouteArgs a, int n_tc) {
  __shared__ float Ms[256], iLs[256];
  const int x = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_trigger();
  pdl_wait();
  const int len = checked_len(a, b, false);
  const bool route = x < n_tc;
  const int h_lo = route ? 0 : (x - n_tc) * G;
  const int h_n = route ? a.Hq : G;
  // sequence-wide (M_h, 1/L_h) from the chunk partials
  for (int hh = warp; hh < h_n; hh += 8) {
    const float2* ml = a.part_ml + ((int64_t)b * a.Hq + h_lo + hh) * a.n_split;
    float M = -INFINITY;
    for (int s = lane; s < a.n_split; s += 32) M = fmaxf(M, ml[s].x);
    M = warp_max(M);
    float L = 0.f;
    for (int s = lane; s < a.n_split; s += 32) {
      const float2 v = ml[s];
      if (v.y > 0.f) L += exp2f(v.x - M) * v.y;
    }
    L = warp_sum(L);
    if (lane == 0) {
      Ms[hh] = M;
      iLs[hh] = L > 0.f ? 1.f / L : 0.f;
    }
  }
  __syncthreads();
  if (route) {
    const int tb = x * kTokPerRouteCta;
    const int te = min(len, tb + kTokPerRouteCta);
    for (int t = tb + tid; t < te; t += 256) {
      float r = 0.f;
      for (int h = 0; h < a.Hq; ++h) r += exp2f(a.z[((int64_t)b * a.Hq + h) * a.zld + t] - Ms[h]) * iLs[h];
      a.scores[(int64_t)b * a.ld + t] = r;
    }
  } else {
    for (int e = tid; e < G * kD; e += 256) {
      const int hh = e / kD, c = e % kD, h = h_lo + hh;
      const float M = Ms[hh];
      const float2* ml = a.part_ml + ((int64_t)b * a.Hq + h) * a.n_split;
      const float* po = a.part_o + ((int64_t)b * a.Hq + h) * a.n_split * kD + c;
      float acc = 0.f;
      for (int s = 0; s < a.n_split; ++s) {
        const float2 v = ml[s];
        if (v.y > 0.f) acc += exp2f(v.x - M) * po[(int64_t)s * kD];
      }
      const float o = acc * iLs[hh];
      const int64_t off = ((int64_t)b * a.Hq + h) * kD + c;
      if (a.out_f32)
        reinterpret_cast<float*>(a.O)[off] = o;
      else
        reinterpret_cast<uint16_t*>(a.O)[off] = __bfloat16_as_ushort(__float2bfloat16_rn(o));
    }
  }
}

template <int G>
cudaError_t launch(const RouteArgs& a, cudaStream_t stream) {
  auto k1 = indexer_layer_partial_kernel<G>;
  cudaError_t e = ensure_smem(k1, PartLayout<G>::kSmem);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)a.n_split, (unsigned)a.Hkv, (unsigned)a.B);
  cfg.blockDim = dim3(kPartThreads);
  cfg.dynamicSmemBytes = PartLayout<G>::kSmem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, k1, a);
  if (e != cudaSuccess) return e;
  const int n_tc = (a.S_max + kTokPerRouteCta - 1) / kTokPerRouteCta;
  cudaLaunchConfig_t cfg2 = cfg;
  cfg2.gridDim = dim3((unsigned)(n_tc + a.Hkv), (unsigned)a.B);
  cfg2.blockDim = dim3(256);
  cfg2.dynamicSmemBytes = 0;
  e = cudaLaunchKernelEx(&cfg2, indexer_layer_combine_kernel<G>, a, n_tc);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

size_t route_ws_bytes(int B, int S_max, int Hq) {
  const size_t n_split = ((size_t)S_max + kRouteChunk - 1) / kRouteChunk;
  const size_t zld = ((size_t)S_max + 63) / 64 * 64;
  auto r256 = [](size_t x) { return (x + 255) / 256 * 256; };
  return r256((size_t)B * Hq * zld * 4) + r256((size_t)B * Hq * n_split * 8) +
         r256((size_t)B * Hq * n_split * kD * 4);
}

cudaError_t launch_indexer_layer_attn(const RouteArgs& a, cudaStream_t stream) {
  switch (a.Hq / a.Hkv) {
    case 1: return launch<1>(a, stream);
    case 2: return launch<2>(a, stream);
    case 4: return launch<4>(a, stream);
    case 8: return launch<8>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace sa
