// Lightning-indexer score on tcgen05 tensor cores.
//
// Definition [IndexCache: Accelerating Sparse Attention via Cross-Layer
// Index Reuse, technical summary section 1: the indexer scores every
// previous token for the current query; CLSA news article, "Comment CLSA
// fonctionne": the shared indexer layer computes the scores once]:
//   score[b,t] = sum_j w[b,j] * max(0, qI[b,j,:] . KI[seq_off[b]+t, :])
//
// Decode form.  The step is HBM-bound: every visible key row (d_I bf16) is
// read once, and each row feeds H_I dot products of length d_I (16 flop per
// byte at H_I=16), above what the fp32 FMA pipes sustain at HBM rate, so the
// contraction runs on the tensor cores:
//   A = 128 key rows x d_I   (TMA, 128-byte swizzle, K-major)
//   B = H_I (padded to N) query heads x d_I (TMA, same layout)
//   D = 128 x N fp32 in TMEM; the epilogue warps read one token per thread,
//       apply ReLU, weight, sum over heads and store one fp32 score.
// Persistent CTAs (one per SM) walk the ragged list of (sequence, 128-token
// tile) pairs; warp 0 issues TMA into a STAGES-deep ring, warp 1 issues the
// MMAs into ACC TMEM accumulators, warps 2-5 run the epilogue.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "indexer.cuh"
#include "sm100.cuh"
#include "timeline.cuh"

namespace sa {
namespace {

constexpr int kTile = 128;
constexpr int kAcc = 4;
constexpr int kThreads = 192;
constexpr int kMaxStages = 4;  // measured: 4 beats 3, 5 and 6 on B200 (more in flight is slower)
constexpr int kSmemMax = 232448;  // dynamic shared memory per CTA on sm_100

// full[kMaxStages] empty[kMaxStages] tfull[kAcc] tempty[kAcc] | tmem slot |
// prefix[B+1] | ring of n_st stages (1024-aligned; as many as fit, up to 6)
constexpr int kBarOffset = 0;
constexpr int kTmemSlotOffset = 8 * (2 * kMaxStages + 2 * kAcc);
constexpr int kPrefixOffset = kTmemSlotOffset + 16;

template <int NHALF, int NPAD>
struct IdxLayout {
  static constexpr int kABytes = NHALF * kTile * 128;
  static constexpr int kBBytes = NHALF * NPAD * 128;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTmemCols = (kAcc * NPAD <= 32) ? 32 : (kAcc * NPAD <= 64) ? 64 : (kAcc * NPAD <= 128) ? 128 : 256;
  static int ring_offset(int B) { return (kPrefixOffset + 4 * (B + 1) + 1023) / 1024 * 1024; }
  static int stages(int B) {
    const int n = (kSmemMax - 1024 - ring_offset(B)) / kStageBytes;
    return n > kMaxStages ? kMaxStages : n;
  }
  static size_t smem_bytes(int B) { return 1024 + (size_t)ring_offset(B) + (size_t)stages(B) * kStageBytes; }
};

__device__ __forceinline__ int locate_tile(const int* prefix, int B, int g) {
  // largest b with prefix[b] <= g (prefix[0] = 0, prefix[B] = total)
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= g) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// One warp, for the new token of sequence b (row len-1 of its caches): copies
// its indexer key and its K / V rows of every KV head into the caches, then
// stores its score computed from the fresh key.  Lane j takes indexer head j
// (and j + 32): its whole dot product, with every load issued before the
// arithmetic, then one butterfly sum of the weighted ReLU terms.  Tiles that
// loaded this row from the cache are not used for it.
__device__ __noinline__ void append_new_token(const AppendArgs& ap, const float* __restrict__ w,
                                              const int64_t* __restrict__ seq_off, int b, int len, int H_I,
                                              int d_I, float* score_out, int lane) {
  const int64_t off = seq_off[b];
  const uint16_t* nk = ap.new_KI + (int64_t)b * d_I;
  uint16_t* kdst = ap.KI + (off + len - 1) * d_I;
  for (int c = lane * 8; c < d_I; c += 256)
    *reinterpret_cast<uint4*>(kdst + c) = *reinterpret_cast<const uint4*>(nk + c);
  if (ap.new_K != nullptr) {
    const int per_row = ap.d / 8;  // 16-byte pieces of a row
    for (int i = lane; i < ap.Hkv * per_row; i += 32) {
      const int h = i / per_row, pc = i % per_row;
      const int64_t row = off * ap.Hkv + (int64_t)h * len + (len - 1);
      const int64_t src = ((int64_t)b * ap.Hkv + h) * ap.d;
      reinterpret_cast<uint4*>(ap.K + row * ap.d)[pc] = reinterpret_cast<const uint4*>(ap.new_K + src)[pc];
      reinterpret_cast<uint4*>(ap.V + row * ap.d)[pc] = reinterpret_cast<const uint4*>(ap.new_V + src)[pc];
    }
  }
  float acc = 0.f;
  for (int j = lane; j < H_I; j += 32) {
    const uint4* q = reinterpret_cast<const uint4*>(ap.qI + ((int64_t)b * H_I + j) * d_I);
    const uint4* k = reinterpret_cast<const uint4*>(nk);
    const float wj = __ldg(&w[(int64_t)b * H_I + j]);
    float dot = 0.f;
    for (int c8 = 0; c8 < d_I / 8; c8 += 4) {  // d_I is a multiple of 64: four 16-byte pieces at a time
      uint4 qv[4], kv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        qv[u] = q[c8 + u];
        kv[u] = k[c8 + u];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t qa[4] = {qv[u].x, qv[u].y, qv[u].z, qv[u].w};
        const uint32_t ka[4] = {kv[u].x, kv[u].y, kv[u].z, kv[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          dot = fmaf(__uint_as_float(qa[e] << 16), __uint_as_float(ka[e] << 16), dot);
          dot = fmaf(__uint_as_float(qa[e] & 0xffff0000u), __uint_as_float(ka[e] & 0xffff0000u), dot);
        }
      }
    }
    acc = fmaf(wj, fmaxf(dot, 0.f), acc);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) *score_out = __fadd_rn(acc, 0.f);  // canonical +0
}

template <int NHALF, int NPAD, bool APPEND>
__global__ void __launch_bounds__(kThreads, 1)
indexer_decode_kernel(const __grid_constant__ CUtensorMap tm_ki, const __grid_constant__ CUtensorMap tm_qi,
                      const float* __restrict__ w, const int64_t* __restrict__ seq_off,
                      const int32_t* __restrict__ seq_len, int B, int64_t n_tokens, int S_max, int H_I,
                      float* __restrict__ scores, int64_t ld, DeviceStatus* __restrict__ status, int n_st,
                      int ring_off, const AppendArgs ap) {
  using Lay = IdxLayout<NHALF, NPAD>;
  const int kStages = n_st;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kBarOffset);
  uint64_t* empty = full + kMaxStages;
  uint64_t* tfull = empty + kMaxStages;
  uint64_t* tempty = tfull + kAcc;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kTmemSlotOffset);
  int* prefix = reinterpret_cast<int*>(smem + kPrefixOffset);
  uint8_t* ring = smem + ring_off;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- set-up: barriers and TMEM (overlaps the previous kernel's tail) ----
  pdl_trigger();
  if (threadIdx.x == 0) SA_TL(kTlIndexer, 0);
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < kStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int a = 0; a < kAcc; ++a) { mbar_init(&tfull[a], 1); mbar_init(&tempty[a], 4); }
    fence_mbar_init();
    tma_prefetch_desc(&tm_ki);
    tma_prefetch_desc(&tm_qi);
  } else if (warp == 1) {
    tmem_alloc(tmem_slot, Lay::kTmemCols);
  }
  // everything below reads what earlier kernels of the stream wrote
  pdl_wait();
  if (warp == 0) {
    // prefix[b] = sum of ceil(len/128) over earlier sequences (warp scan in chunks)
    int carry = 0;
    for (int base = 0; base < B; base += 32) {
      const int b = base + lane;
      int n = 0;
      if (b < B) {
        int len = seq_len[b];
        if (len > S_max || len < 0) {
          report(status, kErrDevice, kKernIndexer, b, len, S_max);
          len = len < 0 ? 0 : S_max;
        }
        n = (len + kTile - 1) / kTile;
      }
      int incl = n;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (b < B) prefix[b] = carry + incl - n;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) prefix[B] = carry;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = prefix[B];
  if (threadIdx.x == 0) SA_TL(kTlIndexer, 1);

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int i = 0;
      for (int g = blockIdx.x; g < total; g += gridDim.x, ++i) {
        const int s = i % kStages;
        if (!mbar_wait(&empty[s], ((i / kStages) & 1) ^ 1, kWaitLimitNs)) {
          report(status, kErrTimeout, kKernIndexer, blockIdx.x, 0, i);
          break;
        }
        const int b = locate_tile(prefix, B, g);
        const int tl = g - prefix[b];
        const int64_t row = seq_off[b] + (int64_t)tl * kTile;
        uint8_t* st = ring + s * Lay::kStageBytes;
        mbar_arrive_expect_tx(&full[s], Lay::kStageBytes);
#pragma unroll
        for (int h = 0; h < NHALF; ++h) tma_load_2d(st + h * kTile * 128, &tm_ki, &full[s], h * 64, (int)row);
#pragma unroll
        for (int h = 0; h < NHALF; ++h)
          tma_load_3d(st + Lay::kABytes + h * NPAD * 128, &tm_qi, &full[s], h * 64, 0, b);
      }
      // drain: every load issued by this thread has landed before the CTA exits
      const int issued = i;
      for (int j = issued - kStages; j < issued; ++j)
        if (j >= 0) mbar_wait(&full[j % kStages], (j / kStages) & 1, kWaitLimitNs);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(128, NPAD, false, false);
      int i = 0;
      for (int g = blockIdx.x; g < total; g += gridDim.x, ++i) {
        const int s = i % kStages;
        const int a = i % kAcc;
        if (!mbar_wait(&full[s], (i / kStages) & 1, kWaitLimitNs) ||
            !mbar_wait(&tempty[a], ((i / kAcc) & 1) ^ 1, kWaitLimitNs)) {
          report(status, kErrTimeout, kKernIndexer, blockIdx.x, 1, i);
          break;
        }
        tc_fence_after();
        const uint32_t a_base = smem_u32(ring + s * Lay::kStageBytes);
        const uint32_t b_base = a_base + Lay::kABytes;
        const uint32_t d = tmem_base + a * NPAD;
#pragma unroll
        for (int h = 0; h < NHALF; ++h) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = umma_desc_sw128(a_base + h * kTile * 128 + kk * 32, 16, 1024);
            const uint64_t bd = umma_desc_sw128(b_base + h * NPAD * 128 + kk * 32, 16, 1024);
            umma_bf16(d, ad, bd, idesc, (h | kk) != 0);
          }
        }
        umma_commit(&empty[s]);
        umma_commit(&tfull[a]);
      }
    }
  } else {
    // ---------------- epilogue: ReLU, head weights, sum ----------------
    const int quarter = warp & 3;  // TMEM lanes this warp may read
    const int r = quarter * 32 + lane;
    int i = 0;
    int cur_b = -1;
    float wr[NPAD];
#pragma unroll
    for (int j = 0; j < NPAD; ++j) wr[j] = 0.f;
    for (int g = blockIdx.x; g < total; g += gridDim.x, ++i) {
      const int a = i % kAcc;
      bool ok = true;  // lane 0 waits for the warp, so a give-up never splits it
      if (lane == 0) ok = mbar_wait(&tfull[a], (i / kAcc) & 1, kWaitLimitNs);
      if (!__shfl_sync(0xffffffffu, ok, 0)) {
        if (lane == 0) report(status, kErrTimeout, kKernIndexer, blockIdx.x, 2, i);
        break;
      }
      tc_fence_after();
      uint32_t v[NPAD];
#pragma unroll
      for (int c = 0; c < NPAD; c += 16)
        tmem_ld16(tmem_base + ((uint32_t)(quarter * 32) << 16) + a * NPAD + c, &v[c]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[a]);

      const int b = locate_tile(prefix, B, g);
      if (b != cur_b) {
        cur_b = b;
#pragma unroll
        for (int j = 0; j < NPAD; ++j) wr[j] = (j < H_I) ? __ldg(&w[(int64_t)b * H_I + j]) : 0.f;
      }
      int len = seq_len[b];
      len = len < 0 ? 0 : (len > S_max ? S_max : len);
      const int t = (g - prefix[b]) * kTile + r;
      // the new token's row, when this call appends it, is scored below from
      // its fresh key (the tile may hold the stale cache row)
      const int t_new = APPEND ? len - 1 : -1;
      if (warp == 2 && lane == 0) SA_TL(kTlIndexer, 2 + (b < 12 ? b : 12));  // this CTA's last tile of b
      if (t < len && t != t_new) {
        float acc = 0.f;
#pragma unroll
        for (int j = 0; j < NPAD; ++j)
          if (j < H_I) acc = fmaf(wr[j], fmaxf(__uint_as_float(v[j]), 0.f), acc);
        scores[(int64_t)b * ld + t] = __fadd_rn(acc, 0.f);  // canonical +0
        if (t == 0 && seq_off[b] + len > n_tokens)
          report(status, kErrDevice, kKernIndexer, b, seq_off[b] + len, n_tokens);
      }
      if (APPEND && t_new >= 0 && t_new / kTile == g - prefix[b] && (t_new % kTile) / 32 == quarter)
        append_new_token(ap, w, seq_off, b, len, H_I, 64 * NHALF, scores + (int64_t)b * ld + t_new, lane);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) SA_TL(kTlIndexer, 15);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Lay::kTmemCols);
  }
}

template <int NHALF, int NPAD>
cudaError_t launch_decode(const IndexerArgs& a, const CUtensorMap& tm_ki, const CUtensorMap& tm_qi,
                          int num_sms, cudaStream_t stream) {
  using Lay = IdxLayout<NHALF, NPAD>;
  // the new-token append is compiled only into the kernel that does it
  auto kern = a.ap.new_KI != nullptr ? indexer_decode_kernel<NHALF, NPAD, true>
                                     : indexer_decode_kernel<NHALF, NPAD, false>;
  const size_t smem = Lay::smem_bytes(a.B);
  cudaError_t e = ensure_smem(kern, smem);
  if (e != cudaSuccess) return e;
  const int64_t tiles_ub = (int64_t)a.B * ((a.S_max + kTile - 1) / kTile);
  int grid = (int)(tiles_ub < num_sms ? tiles_ub : num_sms);
  if (grid < 1) grid = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (Lay::stages(a.B) < 2) return cudaErrorInvalidValue;  // the prefix table would crowd out the ring
  e = cudaLaunchKernelEx(&cfg, kern, tm_ki, tm_qi, a.w, a.seq_off, a.seq_len, a.B, a.n_tokens, a.S_max, a.H_I,
                         a.scores, a.ld, a.status, Lay::stages(a.B), Lay::ring_offset(a.B), a.ap);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_indexer_decode(const IndexerArgs& a, const CUtensorMap& tm_ki, const CUtensorMap& tm_qi,
                                  int npad, int num_sms, cudaStream_t stream) {
  const int nh = a.d_I / 64;
#define SA_IDX_CASE(NH, NP) \
  if (nh == NH && npad == NP) return launch_decode<NH, NP>(a, tm_ki, tm_qi, num_sms, stream);
  SA_IDX_CASE(1, 16) SA_IDX_CASE(1, 32) SA_IDX_CASE(1, 48) SA_IDX_CASE(1, 64)
  SA_IDX_CASE(2, 16) SA_IDX_CASE(2, 32) SA_IDX_CASE(2, 48) SA_IDX_CASE(2, 64)
  SA_IDX_CASE(3, 16) SA_IDX_CASE(3, 32) SA_IDX_CASE(3, 48) SA_IDX_CASE(3, 64)
  SA_IDX_CASE(4, 16) SA_IDX_CASE(4, 32) SA_IDX_CASE(4, 48) SA_IDX_CASE(4, 64)
#undef SA_IDX_CASE
  return cudaErrorInvalidValue;
}

}  // namespace sa

SA_TL_SETTER(sa_timeline_set_indexer)
