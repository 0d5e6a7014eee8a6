// Lightning-indexer score for the queries of a prefill chunk on tcgen05
// tensor cores.
//
// Definition [IndexCache: Accelerating Sparse Attention via Cross-Layer
// Index Reuse, technical summary section 1: the indexer scores every
// previous token for each query; CompactAttention: Accelerating Chunked
// Prefill with Block-Union KV Selection, technical summary "Enonce du
// Probleme": this per-query search, repeated over a whole chunk, is the
// prefill bottleneck]:
//   scores[p, t] = sum_j w[p,j] * max(0, qI[p,j,:] . KI[t,:]),  t <= q_pos[p]
//
// The decode kernel puts one query's H_I heads in the MMA N dimension and
// reads every key row once per query.  Here a CTA owns a block of QB queries
// with QB * H_I = 256 (the largest N of one MMA), so each key tile it streams
// feeds QB queries at once:
//   B = the block's 256 (query, head) rows x d_I, loaded once (TMA, 128-byte
//       swizzle, K-major);
//   A = 128 keys x d_I per stage (TMA ring, keys up to the block's last
//       position);
//   D = 128 x 256 fp32 in TMEM, two accumulators (512 columns);
//   8 epilogue warps: warps w and w+4 read the same 32 TMEM lanes (key rows),
//       one the first 128 columns and one the last; a thread turns its 128
//       values (128/H_I queries x H_I heads) into 128/H_I scores.
// Warp 0 issues TMA, warp 1 owns TMEM and issues the MMAs.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "indexer.cuh"
#include "sm100.cuh"
#include "status.cuh"

namespace sa {
namespace {

constexpr int kTile = 128;     // keys per stage (MMA M)
constexpr int kN = 256;        // (query, head) rows per block (MMA N)
constexpr int kStages = 4;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;

template <int NHALF>  // d_I = 64 * NHALF
struct PfLayout {
  static constexpr int kBBytes = NHALF * kN * 128;     // [NHALF][256 rows][128 B]
  static constexpr int kABytes = NHALF * kTile * 128;  // one key tile
  static constexpr int kBOff = 0;
  static constexpr int kRingOff = kBBytes;
  static constexpr int kWOff = kRingOff + kStages * kABytes;  // w of the block, [256] fp32
  static constexpr int kBarOff = kWOff + kN * 4;              // full[4] empty[4] tfull[2] tempty[2] qbar
  static constexpr int kSlotOff = kBarOff + 8 * (2 * kStages + 4 + 1);
  static constexpr int kMiscOff = kSlotOff + 16;  // [0]: end of the block's key range
  static constexpr int kSmem = 1024 + kMiscOff + 16;
};

template <int NHALF, int HI>
__global__ void __launch_bounds__(kThreads, 1)
indexer_prefill_kernel(const __grid_constant__ CUtensorMap tm_ki, const __grid_constant__ CUtensorMap tm_qi,
                       const float* __restrict__ w, const int32_t* __restrict__ q_pos, int Nq, int S, int max_pos,
                       float* __restrict__ scores, int64_t ld, DeviceStatus* __restrict__ status) {
  using Lay = PfLayout<NHALF>;
  constexpr int QB = kN / HI;    // queries per block
  constexpr int QPT = QB / 2;    // queries per epilogue thread
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* bq = smem + Lay::kBOff;
  uint8_t* ring = smem + Lay::kRingOff;
  float* w_s = reinterpret_cast<float*>(smem + Lay::kWOff);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Lay::kBarOff);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* qbar = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kSlotOff);
  int* misc = reinterpret_cast<int*>(smem + Lay::kMiscOff);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q0 = blockIdx.x * QB;

  // ---- set-up (overlaps the previous kernel's tail), then the inputs ----
  pdl_trigger();
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < kStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&tfull[a], 1); mbar_init(&tempty[a], kEpiWarps); }
    mbar_init(qbar, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_ki);
    tma_prefetch_desc(&tm_qi);
  } else if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
  }
  pdl_wait();
  if (warp == 0) {
    // the block's key range ends after its last query's position
    int hi = -1;
    for (int q = lane; q < QB; q += 32) {
      const int p = q0 + q;
      if (p < Nq) {
        int pos = q_pos[p];
        if (pos < 0 || pos > max_pos) {
          report(status, kErrDevice, kKernIndexerPrefill, p, pos, max_pos);
          pos = pos < 0 ? 0 : max_pos;
        }
        hi = max(hi, pos);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    if (lane == 0) misc[0] = min(hi + 1, S);
  } else if (warp >= 2) {
    for (int i = threadIdx.x - 64; i < kN; i += 32 * kEpiWarps) {
      const int q = q0 + i / HI;
      w_s[i] = q < Nq ? __ldg(&w[(int64_t)q0 * HI + i]) : 0.f;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int kend = misc[0];
  const int ntiles = (kend + kTile - 1) / kTile;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      mbar_arrive_expect_tx(qbar, (uint32_t)Lay::kBBytes);
#pragma unroll
      for (int h = 0; h < NHALF; ++h) tma_load_2d(bq + h * kN * 128, &tm_qi, qbar, h * 64, q0 * HI);
      int i = 0;
      for (; i < ntiles; ++i) {
        const int s = i % kStages;
        if (!mbar_wait(&empty[s], ((i / kStages) & 1) ^ 1, kWaitLimitNs)) {
          report(status, kErrTimeout, kKernIndexerPrefill, blockIdx.x, 0, i);
          break;
        }
        uint8_t* st = ring + s * Lay::kABytes;
        mbar_arrive_expect_tx(&full[s], (uint32_t)Lay::kABytes);
#pragma unroll
        for (int h = 0; h < NHALF; ++h) tma_load_2d(st + h * kTile * 128, &tm_ki, &full[s], h * 64, i * kTile);
      }
      // drain: every load issued by this thread has landed before the CTA exits
      for (int j = i - kStages; j < i; ++j)
        if (j >= 0) mbar_wait(&full[j % kStages], (j / kStages) & 1, kWaitLimitNs);
      mbar_wait(qbar, 0, kWaitLimitNs);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(128, kN, false, false);
      bool ok = ntiles == 0 || mbar_wait(qbar, 0, kWaitLimitNs);
      int i = 0;
      for (; i < ntiles && ok; ++i) {
        const int s = i % kStages, a = i & 1;
        if (!mbar_wait(&full[s], (i / kStages) & 1, kWaitLimitNs) ||
            !mbar_wait(&tempty[a], ((i >> 1) & 1) ^ 1, kWaitLimitNs)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_base = smem_u32(ring + s * Lay::kABytes);
        const uint32_t b_base = smem_u32(bq);
        const uint32_t d = tmem_base + a * kN;
#pragma unroll
        for (int h = 0; h < NHALF; ++h) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = umma_desc_sw128(a_base + h * kTile * 128 + kk * 32, 16, 1024);
            const uint64_t bd = umma_desc_sw128(b_base + h * kN * 128 + kk * 32, 16, 1024);
            umma_bf16(d, ad, bd, idesc, (h | kk) != 0);
          }
        }
        umma_commit(&empty[s]);
        umma_commit(&tfull[a]);
      }
      if (!ok) report(status, kErrTimeout, kKernIndexerPrefill, blockIdx.x, 1, i);
    }
  } else {
    // ---------------- epilogue: ReLU, head weights, sum per query ----------------
    const int ew = warp - 2;
    const int quarter = warp & 3;  // TMEM lanes this warp may read
    const int chalf = ew >> 2;     // columns [128 chalf, +128): queries [QPT chalf, +QPT)
    const int r = quarter * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    for (int i = 0; i < ntiles; ++i) {
      const int a = i & 1;
      bool ok = true;  // lane 0 waits for the warp, so a give-up never splits it
      if (lane == 0) ok = mbar_wait(&tfull[a], (i >> 1) & 1, kWaitLimitNs);
      if (!__shfl_sync(0xffffffffu, ok, 0)) {
        if (lane == 0) report(status, kErrTimeout, kKernIndexerPrefill, blockIdx.x, 2, i);
        break;
      }
      tc_fence_after();
      uint32_t v[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tmem_base + lane_addr + a * kN + chalf * 128 + c * 32, &v[c * 32]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[a]);
      const int t = i * kTile + r;
      if (t < kend) {
#pragma unroll
        for (int qq = 0; qq < QPT; ++qq) {
          const int ql = chalf * QPT + qq;
          float acc = 0.f;
#pragma unroll
          for (int j = 0; j < HI; ++j) acc = fmaf(w_s[ql * HI + j], fmaxf(__uint_as_float(v[qq * HI + j]), 0.f), acc);
          if (q0 + ql < Nq) scores[(int64_t)(q0 + ql) * ld + t] = __fadd_rn(acc, 0.f);  // canonical +0
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

template <int NHALF, int HI>
cudaError_t launch_as(const PrefillIndexerArgs& a, const CUtensorMap& tm_ki, const CUtensorMap& tm_qi,
                      cudaStream_t stream) {
  using Lay = PfLayout<NHALF>;
  auto kern = indexer_prefill_kernel<NHALF, HI>;
  cudaError_t e = ensure_smem(kern, Lay::kSmem);
  if (e != cudaSuccess) return e;
  constexpr int QB = kN / HI;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((a.Nq + QB - 1) / QB));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = Lay::kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, tm_ki, tm_qi, a.w, a.q_pos, a.Nq, a.S, a.max_pos, a.scores, a.ld, a.status);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

bool indexer_prefill_supported(int H_I, int d_I) {
  const bool pow2 = H_I >= 2 && H_I <= 64 && (H_I & (H_I - 1)) == 0;
  return pow2 && (d_I == 64 || d_I == 128);
}

cudaError_t launch_indexer_prefill(const PrefillIndexerArgs& a, const CUtensorMap& tm_ki,
                                   const CUtensorMap& tm_qi, int num_sms, cudaStream_t stream) {
  (void)num_sms;
  if (a.Nq == 0) return cudaSuccess;
  const int nh = a.d_I / 64;
#define SA_PF_CASE(NH, HI) \
  if (nh == NH && a.H_I == HI) return launch_as<NH, HI>(a, tm_ki, tm_qi, stream);
  SA_PF_CASE(1, 2) SA_PF_CASE(1, 4) SA_PF_CASE(1, 8) SA_PF_CASE(1, 16) SA_PF_CASE(1, 32) SA_PF_CASE(1, 64)
  SA_PF_CASE(2, 2) SA_PF_CASE(2, 4) SA_PF_CASE(2, 8) SA_PF_CASE(2, 16) SA_PF_CASE(2, 32) SA_PF_CASE(2, 64)
#undef SA_PF_CASE
  return cudaErrorInvalidValue;
}

}  // namespace sa
