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
// HBM-bound.  A (sequence, KV head) has G = Hq/Hkv query rows (4 or 8 here),
// so every 256-byte K or V row feeds only G dot products of length 128.
//
// Partial kernel: one CTA per (2048-key chunk, KV head, sequence).
//   Warp 8 streams the chunk's K tiles, then its V tiles (128 rows x 128
//   dims, two 64-column TMA boxes, 128-byte swizzle) through a ring.
//   Phase 1 on the tensor cores, as in the decode indexer: warp 9 issues
//   D[128 keys x 16] = K_tile . Q^T (the group's heads padded to N = 16)
//   into one of two TMEM accumulators; warps 0-3 turn a key row each into
//   its G logits (log2 units) in shared memory.
//   Then per head (warp h): the chunk max m, p = 2^(z - m) in place,
//   l = sum p, and z out to global memory for the routing scores.
//   Phase 2 on CUDA cores (a GEMV: G rows): o[h] = sum_t p[h,t] V[t], a
//   thread taking 4 dims of 2 heads over one residue class of the tile's
//   rows; the classes are summed at the end.  Writes (m, l) and o per
//   (head, chunk).
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
constexpr int kTileRows = 128;         // keys per ring tile (the MMA's M)
constexpr int kNPad = 16;              // query heads padded to the MMA's N
constexpr int kCompWarps = 8;          // warps 0-7; 0-3 also read the accumulators
constexpr int kProdWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kPartThreads = 32 * 10;
constexpr int kTileBytes = kTileRows * kD * 2;  // 32 KB: two 64-column swizzled boxes
constexpr int kQBytes = 2 * kNPad * 128;        // 4 KB
constexpr int kTokPerRouteCta = 1024;
constexpr uint32_t kTmemCols = 32;              // two 16-column accumulators

template <int G>
struct PartLayout {
  static constexpr int kStages = G <= 4 ? 2 : 3;                 // two CTAs per SM at G <= 4
  static constexpr int kRingOff = 0;                             // [kStages] tiles, 1024-aligned
  static constexpr int kQOff = kRingOff + kStages * kTileBytes;  // [2 halves][16 rows][128 B]
  static constexpr int kZOff = kQOff + kQBytes;                  // [G][kRouteChunk] fp32: z, then p
  static constexpr int kBarOff = kZOff + G * kRouteChunk * 4;    // full, empty [kStages]; acc_full, acc_empty [2]; q
  static constexpr int kSlotOff = kBarOff + 8 * (2 * kStages + 5);
  static constexpr size_t kSmem = 1024 + kSlotOff + 16;          // + alignment slack
  static_assert(kSmem <= 232448, "shared memory budget");
};

__device__ __forceinline__ void comp_bar() { asm volatile("bar.sync 1, %0;" ::"n"(32 * kCompWarps) : "memory"); }

// lane 0 waits, the outcome is the warp's
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
__global__ void __launch_bounds__(kPartThreads, 1)
indexer_layer_partial_kernel(const RouteArgs a, const __grid_constant__ CUtensorMap tm_k,
                             const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_q) {
  using Lay = PartLayout<G>;
  constexpr int ST = Lay::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem + Lay::kRingOff;
  uint8_t* qt = smem + Lay::kQOff;
  float* zs = reinterpret_cast<float*>(smem + Lay::kZOff);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Lay::kBarOff);
  uint64_t* empty = full + ST;
  uint64_t* acc_full = empty + ST;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* qbar = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kSlotOff);
  int* abort_flag = reinterpret_cast<int*>(smem + Lay::kSlotOff + 4);

  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_trigger();
  if (tid == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);  // the MMA's commit (K tiles) or one compute thread (V tiles)
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
    }
    mbar_init(qbar, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_q);
  }
  if (warp == kMmaWarp) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // everything below reads what earlier kernels of the stream wrote
  pdl_wait();
  const int len = checked_len(a, b, split == 0 && g == 0 && tid == 0);
  const int t0 = split * kRouteChunk;
  const int n = max(0, min(kRouteChunk, len - t0));  // keys of this chunk
  const int nt = (n + kTileRows - 1) / kTileRows;     // K tiles, then as many V tiles
  const int row0 = (int)(a.seq_off[b] * a.Hkv + (int64_t)g * len + t0);
  const int h0 = g * G;

  if (warp == kProdWarp) {
    // ---------------- producer: Q, then K tiles, then V tiles ----------------
    if (lane == 0 && nt > 0) {
      mbar_arrive_expect_tx(qbar, kQBytes);
      tma_load_3d(qt, &tm_q, qbar, 0, h0, b);
      tma_load_3d(qt + kNPad * 128, &tm_q, qbar, 64, h0, b);
      int i = 0;
      for (; i < 2 * nt; ++i) {
        const int s = i % ST;
        if (!mbar_wait(&empty[s], ((i / ST) & 1) ^ 1, kWaitLimitNs)) {
          report(a.status, kErrTimeout, kKernRoute, b, split, i);
          break;
        }
        const int tile = i < nt ? i : i - nt;
        const CUtensorMap* tm = i < nt ? &tm_k : &tm_v;
        uint8_t* st = ring + s * kTileBytes;
        mbar_arrive_expect_tx(&full[s], kTileBytes);
        tma_load_2d(st, tm, &full[s], 0, row0 + tile * kTileRows);
        tma_load_2d(st + kTileBytes / 2, tm, &full[s], 64, row0 + tile * kTileRows);
      }
      // every copy issued lands before the CTA exits
      mbar_wait(qbar, 0, kWaitLimitNs);
      for (int j = max(0, i - ST); j < i; ++j) mbar_wait(&full[j % ST], (j / ST) & 1, kWaitLimitNs);
    }
  } else if (warp == kMmaWarp) {
    // ---------------- phase 1 MMAs: D[128 keys x 16] = K_tile . Q^T ----------------
    if (lane == 0 && nt > 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(kTileRows, kNPad, false, false);
      bool ok = mbar_wait(qbar, 0, kWaitLimitNs);
      for (int j = 0; j < nt && ok; ++j) {
        const int s = j % ST, ac = j & 1;
        ok = mbar_wait(&full[s], (j / ST) & 1, kWaitLimitNs) &&
             mbar_wait(&acc_empty[ac], ((j >> 1) & 1) ^ 1, kWaitLimitNs);
        if (!ok) break;
        tc_fence_after();
        const uint32_t a_base = smem_u32(ring + s * kTileBytes);
        const uint32_t b_base = smem_u32(qt);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = umma_desc_sw128(a_base + h * (kTileBytes / 2) + kk * 32, 16, 1024);
            const uint64_t bd = umma_desc_sw128(b_base + h * kNPad * 128 + kk * 32, 16, 1024);
            umma_bf16(tmem + ac * kNPad, ad, bd, idesc, (h | kk) != 0);
          }
        }
        umma_commit(&empty[s]);      // the K tile may be overwritten once these MMAs are done
        umma_commit(&acc_full[ac]);
      }
      if (!ok) {
        report(a.status, kErrTimeout, kKernRoute, b, split, 3000000);
        atomicExch(abort_flag, 1);
      }
    }
  } else {
    // ---------------- phase 1 epilogue: warps 0-3, one key row per thread ----------------
    if (warp < 4) {
      for (int j = 0; j < nt; ++j) {
        const int ac = j & 1;
        if (!warp_wait(&acc_full[ac], (j >> 1) & 1)) {
          if (lane == 0) {
            report(a.status, kErrTimeout, kKernRoute, b, split, 1000000 + j);
            atomicExch(abort_flag, 1);
          }
          break;
        }
        tc_fence_after();
        uint32_t v[16];
        tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + ac * kNPad, v);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[ac]);
        const int t = j * kTileRows + warp * 32 + lane;
        if (t < n) {
#pragma unroll
          for (int h = 0; h < G; ++h) zs[h * kRouteChunk + t] = __uint_as_float(v[h]) * a.scale_log2;
        }
      }
    }
    comp_bar();
    bool go = *reinterpret_cast<volatile int*>(abort_flag) == 0;

    // ---------------- per head: chunk max, weights in place, sum ----------------
    if (go && warp < G) {
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
    // each tile.  A V row sits in two 128-byte swizzled halves: 16-byte chunk
    // c of row r of a half at r*128 + ((c ^ (r & 7)) * 16).
    constexpr int HP = G < 2 ? G : 2;      // heads per thread
    constexpr int NHS = G / HP;            // head slots
    constexpr int NRG = kCompWarps / NHS;  // row groups (8, 8, 4, 2 for G = 1, 2, 4, 8)
    const int dq4 = tid & 31;
    const int hs = (tid >> 5) % NHS;
    const int rg = (tid >> 5) / NHS;
    const uint32_t vcol = (uint32_t)(dq4 >> 4) * (kTileBytes / 2) + (uint32_t)(dq4 & 1) * 8;
    const uint32_t vchunk = (uint32_t)(dq4 & 15) >> 1;
    float o[HP][4];
#pragma unroll
    for (int x = 0; x < HP; ++x)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[x][e] = 0.f;
    for (int j = 0; go && j < nt; ++j) {
      const int i = nt + j, s = i % ST;
      if (!warp_wait(&full[s], (i / ST) & 1)) {
        if (lane == 0) {
          report(a.status, kErrTimeout, kKernRoute, b, split, 2000000 + j);
          atomicExch(abort_flag, 1);
        }
        go = false;
      } else {
        const int rows = min(kTileRows, n - j * kTileRows);
        const uint8_t* vt = ring + s * kTileBytes + vcol;
        const float* pr = zs + (hs * HP) * kRouteChunk + j * kTileRows;
#pragma unroll 4
        for (int r = rg; r < rows; r += NRG) {
          const uint2 v4 = *reinterpret_cast<const uint2*>(vt + r * 128 + ((vchunk ^ (uint32_t)(r & 7)) << 4));
          const float v[4] = {__uint_as_float(v4.x << 16), __uint_as_float(v4.x & 0xffff0000u),
                              __uint_as_float(v4.y << 16), __uint_as_float(v4.y & 0xffff0000u)};
#pragma unroll
          for (int x = 0; x < HP; ++x) {
            const float p = pr[x * kRouteChunk + r];
#pragma unroll
            for (int e = 0; e < 4; ++e) o[x][e] = fmaf(p, v[e], o[x][e]);
          }
        }
      }
      // every compute warp is done with this V tile (or gave up): one arrival frees it
      comp_bar();
      if (tid == 0) mbar_arrive(&empty[s]);
      go = go && *reinterpret_cast<volatile int*>(abort_flag) == 0;
    }
    // sum the row groups (the weights are no longer needed: reuse their space)
    comp_bar();
    go = *reinterpret_cast<volatile int*>(abort_flag) == 0;
    float* red = zs;  // [NRG][G][128]
    if (go) {
#pragma unroll
      for (int x = 0; x < HP; ++x)
        *reinterpret_cast<float4*>(red + ((rg * G) + hs * HP + x) * kD + 4 * dq4) =
            make_float4(o[x][0], o[x][1], o[x][2], o[x][3]);
    }
    comp_bar();
    if (go) {
      for (int e = tid; e < G * kD; e += 32 * kCompWarps) {
        float sum = 0.f;
#pragma unroll
        for (int q = 0; q < NRG; ++q) sum += red[q * G * kD + e];
        a.part_o[(((int64_t)b * a.Hq + h0 + e / kD) * a.n_split + split) * kD + e % kD] = sum;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
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
cudaError_t launch(const RouteArgs& a, const CUtensorMap& tm_k, const CUtensorMap& tm_v, const CUtensorMap& tm_q,
                   cudaStream_t stream) {
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
  e = cudaLaunchKernelEx(&cfg, k1, a, tm_k, tm_v, tm_q);
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

cudaError_t launch_indexer_layer_attn(const RouteArgs& a, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                                      const CUtensorMap& tm_q, cudaStream_t stream) {
  switch (a.Hq / a.Hkv) {
    case 1: return launch<1>(a, tm_k, tm_v, tm_q, stream);
    case 2: return launch<2>(a, tm_k, tm_v, tm_q, stream);
    case 4: return launch<4>(a, tm_k, tm_v, tm_q, stream);
    case 8: return launch<8>(a, tm_k, tm_v, tm_q, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace sa
