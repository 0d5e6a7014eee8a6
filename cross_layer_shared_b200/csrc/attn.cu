// Gather-based sparse softmax attention on tcgen05 tensor cores.
//
// Decode [IndexCache technical summary section 1: main attention runs over
// the k selected tokens only; section 2: S layers reuse the index of the
// nearest upstream F layer; CLSA news article "Comment CLSA fonctionne":
// one index is handed to every cross-decoder layer over the shared KV
// cache].  All layers of a group read the same selected K/V rows, so one
// CTA stacks the queries of every layer and every head of a GQA group into
// the M rows of one MMA tile (row r = layer r/G, head g*G + r%G) and gathers
// each selected K/V row from HBM once for all of them.
//
// Chunked prefill [CompactAttention technical summary, execution step: the
// union block table is read in place, no compaction copy]: the same kernel
// with rows = (query, head of the group), keys = the tokens of the group's
// union blocks, and a causal limit per row.
//
// Per CTA (384 threads, warp-specialised):
//   warps 9-11  gather 128 K rows and 128 V rows per tile with TMA
//               (tile::gather4: 4 rows x 128 bytes per instruction) into
//               128-byte swizzled shared memory, a 3-deep ring (2 in the
//               precise-P variant); each warp signals its bytes on the
//               stage's mbarrier; the next tile's indices load early;
//   warp 8      owns TMEM (512 columns: S double buffer, O0, O1) and issues
//               S = Q K^T (M=128 rows, N=128 keys, K=d=128) and, per key
//               half h, O_h += P_h V_h (V read MN-major), so the next
//               tile's QK^T overlaps this tile's softmax;
//   warps 0-7   softmax: warp w owns rows 32(w%4).. and key half w/4, one
//               row per thread, with its own running max / sum / O_h (exp2
//               domain, lazy rescale: O_h is rescaled only when the max
//               grows by more than 2^8); P in bf16 (or a hi+lo bf16 pair for
//               fp32 outputs) written over the consumed K tile.
//   The two halves are merged at the end; key splits of one row tile run as
//   a thread-block cluster: each CTA stages its (m, l, O) per output slice
//   and bulk-copies slice t into CTA t's shared memory, which merges it.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "attn.cuh"
#include "sm100.cuh"
#include "timeline.cuh"

namespace sa {
namespace {

constexpr int kD = 128;
constexpr int kKT = 128;  // keys per tile
constexpr int kSoftWarps = 8;
constexpr int kMmaWarp = 8;
constexpr int kProdWarp0 = 9;  // warps 9, 10, 11
constexpr int kAttnThreads = 384;
constexpr int kMlxOff = 188 * 1024;  // half-merge exchange, past every epilogue slot

template <bool PRECISE>
struct AttnLayout {
  static constexpr int kStages = PRECISE ? 2 : 3;
  static constexpr int kHalf = 16384;  // 128 rows x 128 bytes
  static constexpr int kTile = 2 * kHalf;
  static constexpr int kQOff = 0;
  static constexpr int kStageOff = kTile;
  static constexpr int kStageBytes = 2 * kTile;  // K then V
  static constexpr int kPloOff = kStageOff + kStages * kStageBytes;
  // per stage: 4 validity words (bit c: key 32w+c is real) and the position of
  // key 32w of each word (positions inside a 32-key word are consecutive in prefill)
  static constexpr int kMaskOff = kPloOff + (PRECISE ? 2 * kTile : 0);
  static constexpr int kBarOff = kMaskOff + kStages * 8 * 4;
  // kv_full[ST] kv_empty[ST] s_full[2] s_free[2] p_full[2] o_done[4] recv
  static constexpr int kNBar = 2 * kStages + 11;
  static constexpr int kSlotOff = kBarOff + 8 * kNBar;
  static constexpr size_t kSmem = 1024 + kSlotOff + 16;
  static_assert(kSmem <= 232448, "shared memory budget");
  // ordered skipping: half 1's (log2 tile mass, log2 running mass) per row
  // [128] float2, the votes [kOskSlots tiles][4 warps], then the mbarriers
  // xfull, xfree and dec[kOskSlots].  The producer reads the vote on tile
  // j - kOskSlots before it issues tile j (the softmax and MMA warps read
  // the vote on tile j - 3), so a vote's slot is free again once tile
  // j + kOskSlots can be issued.
  static constexpr int kOskSlots = 3 + kStages;
  static constexpr int kOskOff = (kSlotOff + 16 + 15) & ~15;
  static constexpr int kOskVoteOff = kOskOff + 128 * 8;
  static constexpr int kOskBarOff = kOskVoteOff + kOskSlots * 4 * 4;
  static constexpr size_t kSmemOsk = 1024 + kOskBarOff + (2 + kOskSlots) * 8;
  static_assert(kSmemOsk <= 232448, "shared memory budget (ordered skipping)");
};

// 2^x on the special-function unit (ex2.approx.ftz.f32; 2^-inf = +0)
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// two fp32 values rounded to bf16 (nearest even) and packed, lo in bits 0-15,
// in one conversion instruction
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float bf16_round(float x) { return __bfloat162float(__float2bfloat16_rn(x)); }

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ float4 ld_shared_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Bulk copy of `bytes` from this CTA's shared memory to the same-offset
// layout in CTA `rank` of the cluster, completion counted on that CTA's
// mbarrier (both given as this CTA's addresses, mapped with mapa).
__device__ __forceinline__ void bulk_copy_to_peer(uint32_t dst_local, uint32_t src_local, uint32_t bytes,
                                                  uint64_t* bar_local, int rank) {
  uint32_t dst, bar;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(dst) : "r"(dst_local), "r"(rank));
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(bar) : "r"(smem_u32(bar_local)), "r"(rank));
  asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "r"(src_local), "r"(bytes), "r"(bar)
               : "memory");
}

// A wait whose outcome is the same for every lane of the warp (lane 0 waits,
// the result is broadcast), so that a wait that gives up never splits a warp
// that is about to execute warp-collective instructions.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, kWaitLimitNs);
  return __shfl_sync(0xffffffffu, ok, 0);
}

struct RowMap {
  bool valid;
  int64_t qoff;  // element offset of the row in Q and O
  int limit;     // last visible key position
};

__device__ __forceinline__ RowMap map_row(const AttnArgs& a, int b, int g, int r) {
  RowMap m{false, 0, 0x7FFFFFFF};
  if (r >= a.R) return m;
  m.valid = true;
  const int h = g * a.G + r % a.G;
  if (!a.prefill) {
    const int l = r / a.G;
    m.qoff = (((int64_t)l * a.B + b) * a.Hq + h) * kD;
  } else {
    const int p = r / a.G;
    m.qoff = ((int64_t)p * a.Hq + h) * kD;
    m.limit = a.q_pos[p];
  }
  return m;
}

// row of Q (as a 2-D [rows, d] tensor) holding query row r of (b, g)
__device__ __forceinline__ int q_row(const AttnArgs& a, int b, int g, int r) {
  const int h = g * a.G + r % a.G;
  return a.prefill ? (r / a.G) * a.Hq + h : ((r / a.G) * a.B + b) * a.Hq + h;
}

struct KeySrc {
  int len;   // decode: seq_len[b]
  int base;  // prefill: kv_indptr[g]
  const int32_t* list;  // prefill: the blocks in the order they are read
  int kbeg, kend;
};

// Raw list entry jj (a token index in decode, a block id in prefill), loaded
// without looking at it so that several loads can be in flight; -1 past the
// split's end.  key_fix turns it into a key position, or -1 when the entry is
// padding / invalid (an index past the sequence is reported and skipped).
__device__ __forceinline__ int key_raw(const AttnArgs& a, const KeySrc& ks, int b, int jj) {
  if (jj >= ks.kend) return -1;
  return a.prefill ? __ldg(&ks.list[jj / a.block]) : __ldg(&a.idx[(int64_t)b * a.k + jj]);
}

__device__ __forceinline__ int key_fix(const AttnArgs& a, const KeySrc& ks, int b, int jj, int raw, bool rep) {
  if (jj >= ks.kend || raw < 0) return -1;
  if (!a.prefill) {
    if (raw >= ks.len) {
      if (rep) report(a.status, kErrDevice, kKernAttn, (int64_t)b * a.k + jj, raw, ks.len);
      return -1;
    }
    return raw;
  }
  const int t = raw * a.block + jj % a.block;
  return t < a.S ? t : -1;
}

// n (a multiple of 4) output values of one row, at element offset off of O
__device__ __forceinline__ void store_out(const AttnArgs& a, int64_t off, const float* f, int n) {
  if (a.out_f32) {
    float4* o = reinterpret_cast<float4*>(reinterpret_cast<float*>(a.O) + off);
    for (int e = 0; e < n / 4; ++e) o[e] = make_float4(f[4 * e], f[4 * e + 1], f[4 * e + 2], f[4 * e + 3]);
  } else {
    uint2* o = reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(a.O) + off);
    for (int e = 0; e < n / 4; ++e) o[e] = make_uint2(pack_bf16(f[4 * e], f[4 * e + 1]), pack_bf16(f[4 * e + 2], f[4 * e + 3]));
  }
}

template <bool PRECISE, bool OSK>
__global__ void __launch_bounds__(kAttnThreads, 1)
sparse_attn_kernel(const AttnArgs a, const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v) {
  using Lay = AttnLayout<PRECISE>;
  constexpr int ST = Lay::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint32_t* kmask = reinterpret_cast<uint32_t*>(smem + Lay::kMaskOff);  // [ST][8]
  uint64_t* kv_full = reinterpret_cast<uint64_t*>(smem + Lay::kBarOff);
  uint64_t* kv_empty = kv_full + ST;
  uint64_t* s_full = kv_empty + ST;
  uint64_t* s_free = s_full + 2;
  uint64_t* p_full = s_free + 2;
  uint64_t* o_done = p_full + 2;  // [4]: completion of PV_i on o_done[i % 4]
  uint64_t* recv_bar = o_done + 4;
  uint32_t* slot = reinterpret_cast<uint32_t*>(smem + Lay::kSlotOff);
  // ordered skipping: the row exchange between key halves, the votes, and
  // their barriers (xfull: half 1 wrote, xfree: half 0 read, dec[t % slots]:
  // the four row warps voted on tile t)
  constexpr int kSlots = Lay::kOskSlots;
  float2* osk_x = reinterpret_cast<float2*>(smem + Lay::kOskOff);
  volatile uint32_t* osk_vote = reinterpret_cast<volatile uint32_t*>(smem + Lay::kOskVoteOff);
  uint64_t* osk_xfull = reinterpret_cast<uint64_t*>(smem + Lay::kOskBarOff);
  uint64_t* osk_xfree = osk_xfull + 1;
  uint64_t* osk_dec = osk_xfull + 2;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int u = blockIdx.x;
  const int split = u % a.n_split;
  const int mt = (u / a.n_split) % a.n_mtiles;
  const int bg = u / (a.n_split * a.n_mtiles);
  const int b = a.prefill ? 0 : bg / a.Hkv;
  const int g = a.prefill ? bg : bg % a.Hkv;

  pdl_trigger();
  if (tid == 0) SA_TL(kTlAttn, 0);
  if (warp == kMmaWarp) tmem_alloc(slot, 512);
  if (tid == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    for (int s = 0; s < ST; ++s) {
      mbar_init(&kv_full[s], 3);  // one arrival (with its byte count) per producer warp
      mbar_init(&kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], kSoftWarps);
      mbar_init(&p_full[i], kSoftWarps);
    }
    for (int i = 0; i < 4; ++i) mbar_init(&o_done[i], 1);
    mbar_init(recv_bar, 1);
    if constexpr (OSK) {
      mbar_init(osk_xfull, 4);
      mbar_init(osk_xfree, 4);
      for (int i = 0; i < kSlots; ++i) mbar_init(&osk_dec[i], 4);
    }
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  if (tid == 0) SA_TL(kTlAttn, 1);

  // everything below reads what earlier kernels of the stream wrote
  pdl_wait();
  if (tid == 0) SA_TL(kTlAttn, 2);
  KeySrc ks;
  int n_keys;
  if (!a.prefill) {
    ks.len = a.seq_len[b];
    ks.base = 0;
    ks.list = nullptr;
    n_keys = a.k;
    if (a.idx_count != nullptr) {
      const int c = a.idx_count[b];
      n_keys = c < 0 ? 0 : (c < a.k ? c : a.k);
    }
  } else {
    ks.len = a.S;
    ks.base = a.kv_indptr[g];
    ks.list = OSK ? a.osk_order + (int64_t)mt * a.osk_ld : a.kv_indices + ks.base;
    n_keys = (a.kv_indptr[g + 1] - ks.base) * a.block;
  }
  // decode: the host's even split of k; prefill, and decode with a count of
  // real entries: the size is known only here, so the split is even over it
  // (whole 128-key tiles)
  const int per = (a.prefill || a.idx_count != nullptr)
                      ? ((n_keys + a.n_split - 1) / a.n_split + kKT - 1) / kKT * kKT
                      : a.keys_per_split;
  ks.kbeg = split * per;
  ks.kend = min(n_keys, ks.kbeg + per);
  const int nt = ks.kend > ks.kbeg ? (ks.kend - ks.kbeg + kKT - 1) / kKT : 0;
  int n_run = nt;  // tiles this role runs: nt, or fewer once ordered skipping stops

  // Ordered skipping: whether the vote on tile t says stop (every row's
  // share below tau); the tiles then end after tile t + 2 (the two tiles
  // after it were already in flight), so the softmax and MMA warps read the
  // vote on tile j - 3 before tile j.  ok = false when the wait gave up.
  // One thread, then a whole warp.
  auto osk_vote_stop = [&](int t, bool& ok) -> bool {
    const int sl = t % kSlots;
    ok = mbar_wait(&osk_dec[sl], (t / kSlots) & 1, kWaitLimitNs);
    if (!ok) return false;
    uint32_t any = 0;
#pragma unroll
    for (int w = 0; w < 4; ++w) any |= osk_vote[sl * 4 + w] & 1u;
    return any == 0;
  };
  auto osk_vote_stop_warp = [&](int t, bool& ok) -> bool {
    bool st = false, k2 = true;
    if (lane == 0) st = osk_vote_stop(t, k2);
    ok = __shfl_sync(0xffffffffu, k2, 0);
    return __shfl_sync(0xffffffffu, st, 0);
  };
  // The softmax warps read the vote on tile j - 3 at the top of tile j
  // without waiting on its barrier: a half-1 warp there has passed xfree of
  // tile j - 2, and a half-0 warp xfull of tile j - 1, which the half-0
  // warps reach only after voting on tile j - 3 (each barrier wait is an
  // acquire of every earlier write of the arriving threads).
  auto osk_vote_read_warp = [&](int t) -> bool {
    uint32_t any = 0;
    if (lane == 0) {
      uint32_t v0, v1, v2, v3;
      asm volatile("ld.volatile.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(v0), "=r"(v1), "=r"(v2), "=r"(v3)
                   : "r"(smem_u32(const_cast<uint32_t*>(osk_vote + (t % kSlots) * 4))));
      any = (v0 | v1 | v2 | v3) & 1u;
    }
    return __shfl_sync(0xffffffffu, any, 0) == 0;
  };

  // producer lanes: raw entries of tile rows 4*lane .. 4*lane+3 of the next
  // kPre tiles, all loads in flight at once (a ring in registers, slot = tile
  // % kPre, statically indexed by the unrolled issue loop below).  One tile
  // ahead, every tile's issue waited a whole load latency for its entries.
  constexpr int kPre = 1;
  int raw[kPre][4];
  if (warp >= kProdWarp0) {
#pragma unroll
    for (int t = 0; t < kPre; ++t)
#pragma unroll
      for (int i = 0; i < 4; ++i) raw[t][i] = key_raw(a, ks, b, ks.kbeg + t * kKT + 4 * lane + i);
  }

  // softmax state: thread (row r, key half h)
  const int half = (warp >> 2) & 1;
  const int r_loc = (warp & 3) * 32 + lane;
  const RowMap me = map_row(a, b, g, mt * 128 + r_loc);
  const bool warp_active = warp < kSoftWarps && mt * 128 + (warp & 3) * 32 < a.R;
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
  const uint32_t tmem_oh = tmem + 256 + 128 * half;  // this half's O accumulator
  float m_ref = -INFINITY, l_run = 0.f;
  bool have_o = false;

  if (warp >= kProdWarp0) {
    // =============== producer warps: TMA gathers of K/V (and Q) rows ===============
    // warp 9: K columns 0-63 (+ validity words); warp 10: K columns 64-127
    // (+ Q columns 0-63 on the first tile); warp 11: V columns 0-63 (+ Q
    // columns 64-127 on the first tile); V columns 64-127 split between them.
    const int pw = warp - kProdWarp0;
    const int64_t row_base = a.prefill ? (int64_t)g * a.S : a.seq_off[b] * a.Hkv + (int64_t)g * ks.len;
    bool stop = false;
    // ordered skipping: the producer reads the vote on tile j - kSlots before
    // issuing tile j, far enough back that the vote is in long before the
    // stage is free; tiles issued past the end are drained below
    int issued = nt;       // tiles issued
    int osk_read = 0;      // votes read so far (tiles 0 .. osk_read-1 said continue)
    int osk_n = nt;        // tiles the other roles run, once a stop vote is read
    bool osk_failed = false;
    for (int j0 = 0; j0 < nt && !stop; j0 += kPre) {
#pragma unroll
    for (int jj = 0; jj < kPre; ++jj) {
      const int j = j0 + jj;
      if (j >= nt) break;
      if constexpr (OSK) {
        if (j >= kSlots) {
          bool ok3;
          const bool st3 = osk_vote_stop_warp(j - kSlots, ok3);
          osk_read = j - kSlots + 1;
          if (!ok3) {
            if (lane == 0) report(a.status, kErrTimeout, kKernAttn, u, 5, j);
            osk_failed = true;
            issued = j;
            stop = true;
            break;
          }
          if (st3) {
            osk_n = j - kSlots + 3;
            issued = j;
            stop = true;
            break;
          }
        }
      }
      const int s = j % ST;
      int tc[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) tc[i] = key_fix(a, ks, b, ks.kbeg + j * kKT + 4 * lane + i, raw[jj][i], pw == 0);
#pragma unroll
      for (int i = 0; i < 4; ++i) raw[jj][i] = key_raw(a, ks, b, ks.kbeg + (j + kPre) * kKT + 4 * lane + i);
      bool ok = true;
      if (j >= ST && lane == 0) ok = mbar_wait(&kv_empty[s], ((j / ST) & 1) ^ 1, kWaitLimitNs);
      if (!__shfl_sync(0xffffffffu, ok, 0)) {
        if (lane == 0) report(a.status, kErrTimeout, kKernAttn, u, 0, j);
        issued = j;
        osk_failed = true;
        stop = true;
        break;
      }
      if (pw == 0) {
        // validity words (keys 32w..32w+31 are entries 4l+i of lanes 8w..8w+7)
        // and the position of each word's first key
        uint32_t bal[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) bal[i] = __ballot_sync(0xffffffffu, tc[i] >= 0);
        if (lane < 4) {
          uint32_t word = 0;
#pragma unroll
          for (int l8 = 0; l8 < 8; ++l8)
#pragma unroll
            for (int i = 0; i < 4; ++i) word |= ((bal[i] >> (8 * lane + l8)) & 1u) << (4 * l8 + i);
          kmask[s * 8 + lane] = word;
        }
        if ((lane & 7) == 0) kmask[s * 8 + 4 + (lane >> 3)] = (uint32_t)tc[0];
        __syncwarp();
      }
      // decode: the three warps gather (K lo, V hi), (K hi), (V lo) rows;
      // prefill: the tile is two whole KV blocks, eight 64 x 64 tile loads
      // issued by warp 9 (a block past the list reads rows past the tensor:
      // zeros, so the masked rows of the MMA stay finite)
      // decode: V columns 64-127 are split over the three warps by row group
      // (lanes [vlo, vhi)), so each issues about 43 gathers per tile
      const int vlo = pw == 0 ? 0 : (pw == 1 ? 10 : 21), vhi = pw == 0 ? 10 : (pw == 1 ? 21 : 32);
      const uint32_t tx = (a.prefill ? (pw == 0 ? 2 * Lay::kTile : 0) : Lay::kHalf + (uint32_t)(vhi - vlo) * 512u) +
                          (j == 0 && pw > 0 ? Lay::kHalf : 0);
      if (lane == 0) mbar_arrive_expect_tx(&kv_full[s], tx);
      if (pw == 0 && lane == 0 && j < 8) SA_TL(kTlAttn, 3 + j);  // tile j issued
      __syncwarp();
      const uint32_t kst0 = sbase + Lay::kStageOff + s * Lay::kStageBytes;
      if (a.prefill) {
        if (pw == 0 && lane == 0) {
#pragma unroll
          for (int b2 = 0; b2 < 2; ++b2) {
            const int jj = ks.kbeg + j * kKT + b2 * 64;  // first entry of the block
            const int row = jj < ks.kend ? (int)(row_base + (int64_t)ks.list[jj / 64] * 64)
                                         : a.Hkv * a.S;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              tma_load_2d_u32(kst0 + h * Lay::kHalf + b2 * 8192, &tm_k, &kv_full[s], h * 64, row);
              tma_load_2d_u32(kst0 + Lay::kTile + h * Lay::kHalf + b2 * 8192, &tm_v, &kv_full[s], h * 64, row);
            }
          }
        }
      } else {
        int rk[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) rk[i] = (int)(row_base + (tc[i] < 0 ? 0 : tc[i]));
        const uint32_t kst = kst0 + 4 * lane * 128;
        const uint32_t vst = kst + Lay::kTile;
        if (pw == 0)
          tma_gather4(kst, &tm_k, &kv_full[s], 0, rk);
        else if (pw == 1)
          tma_gather4(kst + Lay::kHalf, &tm_k, &kv_full[s], 64, rk);
        else
          tma_gather4(vst, &tm_v, &kv_full[s], 0, rk);
        if (lane >= vlo && lane < vhi) tma_gather4(vst + Lay::kHalf, &tm_v, &kv_full[s], 64, rk);
      }
      if (j == 0 && pw > 0) {
        int rq[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = mt * 128 + 4 * lane + i;
          rq[i] = q_row(a, b, g, r < a.R ? r : mt * 128);
        }
        tma_gather4(sbase + Lay::kQOff + (pw - 1) * Lay::kHalf + 4 * lane * 128, &tm_q, &kv_full[0], (pw - 1) * 64,
                    rq);
      }
    }
    }
    if constexpr (OSK) {
      // the rest of the votes that can end the tiles before the last issued
      // one, then wait for the issued tiles nobody will consume (their TMA
      // writes land in this CTA's shared memory)
      if (!osk_failed && osk_n == nt) {
        for (int t = osk_read; t + 3 < issued; ++t) {
          bool ok3;
          const bool st3 = osk_vote_stop_warp(t, ok3);
          if (!ok3) {
            if (lane == 0) report(a.status, kErrTimeout, kKernAttn, u, 6, t);
            osk_failed = true;
            break;
          }
          if (st3) {
            osk_n = t + 3;
            break;
          }
        }
      }
      if (!osk_failed)
        for (int t = osk_n; t < issued; ++t)
          if (!warp_wait(&kv_full[t % ST], (t / ST) & 1)) {
            if (lane == 0) report(a.status, kErrTimeout, kKernAttn, u, 7, t);
            break;
          }
    }
  } else if (warp == kMmaWarp) {
    // ======================= MMA issuer =======================
    if (lane == 0) {
      constexpr uint32_t idesc_qk = umma_idesc_bf16(128, 128, false, false);
      constexpr uint32_t idesc_pv = umma_idesc_bf16(128, 128, false, true);
      auto pv = [&](int i) -> bool {
        if (!mbar_wait(&p_full[i & 1], (i >> 1) & 1, kWaitLimitNs)) return false;
        tc_fence_after();
        const uint32_t kst = sbase + Lay::kStageOff + (i % ST) * Lay::kStageBytes;  // P lives here now
        const uint32_t vst = kst + Lay::kTile;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {  // keys 64h + 16kk .. +15
            const uint64_t vd = umma_desc_sw128(vst + h * 8192 + kk * 2048, Lay::kHalf, 1024);
            umma_bf16(tmem + 256 + 128 * h, umma_desc_sw128(kst + h * Lay::kHalf + kk * 32, 16, 1024), vd, idesc_pv,
                      (i | kk) != 0);
            if constexpr (PRECISE)
              umma_bf16(tmem + 256 + 128 * h,
                        umma_desc_sw128(sbase + Lay::kPloOff + (i & 1) * Lay::kTile + h * Lay::kHalf + kk * 32, 16,
                                        1024),
                        vd, idesc_pv, 1);
          }
        }
        umma_commit(&kv_empty[i % ST]);
        umma_commit(&o_done[i & 3]);
        return true;
      };
      bool ok = true;
      for (int j = 0; j < nt && ok; ++j) {
        const int s = j % ST, sb = j & 1;
        ok = mbar_wait(&kv_full[s], (j / ST) & 1, kWaitLimitNs) &&
             mbar_wait(&s_free[sb], ((j >> 1) & 1) ^ 1, kWaitLimitNs);
        if (!ok) break;
        if constexpr (OSK) {
          // S buffer sb free again means every softmax warp is done with
          // tile j - 2, and the half-0 warps voted on tile j - 3 before
          // that: the vote is read without a wait.  A tile the producer
          // issued and this warp does not consume is drained there.
          if (j >= 3) {
            uint32_t any = 0;
#pragma unroll
            for (int w = 0; w < 4; ++w) any |= osk_vote[((j - 3) % kSlots) * 4 + w] & 1u;
            if (any == 0) {
              n_run = j;
              break;
            }
          }
        }
        tc_fence_after();
        const uint32_t kst = sbase + Lay::kStageOff + s * Lay::kStageBytes;
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16(tmem + sb * 128, umma_desc_sw128(sbase + Lay::kQOff + h * Lay::kHalf + kk * 32, 16, 1024),
                      umma_desc_sw128(kst + h * Lay::kHalf + kk * 32, 16, 1024), idesc_qk, (h | kk) != 0);
        umma_commit(&s_full[sb]);
        if (j >= 1) ok = pv(j - 1);
      }
      if (ok && n_run >= 1) ok = pv(n_run - 1);
      if (!ok) report(a.status, kErrTimeout, kKernAttn, u, 1, 0);
    }
  } else {
    // ======================= softmax (warps 0-7) =======================
    bool failed = false;
    for (int j = 0; j < nt; ++j) {
      if constexpr (OSK) {
        if (j >= 3 && osk_vote_read_warp(j - 3)) {
          n_run = j;
          break;
        }
      }
      float tile_sum = 0.f;  // this thread's weights of the tile (relative to m_ref)
      const int s = j % ST, sb = j & 1;
      if (!warp_wait(&s_full[sb], (j >> 1) & 1)) { failed = true; break; }
      if (tid == 0 && j < 8) SA_TL(kTlAttn, 12 + j);  // S of tile j ready
      tc_fence_after();
      if (warp_active) {
        if (!warp_wait(&kv_full[s], (j / ST) & 1)) { failed = true; break; }
        // keys of this half this row may see: the real ones, and in prefill
        // those at or before the row's position (positions are consecutive
        // inside a 32-key word)
        uint32_t vis[2];
#pragma unroll
        for (int w2 = 0; w2 < 2; ++w2) {
          uint32_t v = me.valid ? kmask[s * 8 + 2 * half + w2] : 0u;
          if (a.prefill && v) {
            const int first = (int)kmask[s * 8 + 4 + 2 * half + w2];
            const int room = me.limit - first;  // keys first..first+room are visible
            v &= room >= 31 ? 0xffffffffu : (room < 0 ? 0u : ((2u << room) - 1u));
          }
          vis[w2] = v;
        }
        const bool all_vis = (vis[0] & vis[1]) == 0xffffffffu;
        uint32_t sv[64];
        tmem_ld32(tmem + sb * 128 + 64 * half + lane_base, sv);
        tmem_ld32(tmem + sb * 128 + 64 * half + 32 + lane_base, sv + 32);
        tmem_wait_ld();
        // row maximum over the visible keys: eight independent chains
        float mx[8];
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) mx[c8] = -INFINITY;
        if (all_vis) {
#pragma unroll
          for (int e = 0; e < 64; ++e) mx[e & 7] = fmaxf(mx[e & 7], __uint_as_float(sv[e]));
        } else {
#pragma unroll
          for (int e = 0; e < 64; ++e)
            if ((vis[e >> 5] >> (e & 31)) & 1u) mx[e & 7] = fmaxf(mx[e & 7], __uint_as_float(sv[e]));
        }
        float tmax = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
        tmax *= a.scale_log2;
        float alpha = 1.f;
        bool rescale = false;
        if (j == 0) {
          m_ref = tmax;
        } else if (tmax > m_ref + 8.f) {
          alpha = ex2_approx(m_ref - tmax);
          m_ref = tmax;
          rescale = true;
        }
        l_run *= alpha;
        if (__any_sync(0xffffffffu, rescale)) {
          // O_h is about to be rescaled: the previous tile's PV must have landed.
          // (Its P_lo buffer is never rewritten before then either: PV_{j-2}
          // precedes S_j in the in-order tensor pipe.)
          if (!warp_wait(&o_done[(j - 1) & 3], ((j - 1) >> 2) & 1)) { failed = true; break; }
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t ov[32];
            tmem_ld32(tmem_oh + lane_base + c * 32, ov);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
            tmem_st32(tmem_oh + lane_base + c * 32, ov);
          }
          tmem_wait_st();
        }
        // p = 2^(s*scale*log2e - m_ref), bf16, over this half of the used K tile
        const float neg_m = (m_ref == -INFINITY) ? 0.f : -m_ref;
        const uint32_t pst = sbase + Lay::kStageOff + s * Lay::kStageBytes + half * Lay::kHalf;
        float ls[4] = {0.f, 0.f, 0.f, 0.f};  // four partial sums: short add chains
#pragma unroll
        for (int c16 = 0; c16 < 8; ++c16) {
          float p[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int col = c16 * 8 + e;
            p[e] = ex2_approx(fmaf(__uint_as_float(sv[col]), a.scale_log2, neg_m));
            if (!all_vis && !((vis[col >> 5] >> (col & 31)) & 1u)) p[e] = 0.f;
            ls[e & 3] += p[e];
          }
          const uint32_t off = sw128_offset(r_loc, c16);
          st_shared_v4(pst + off, pack_bf16(p[0], p[1]), pack_bf16(p[2], p[3]), pack_bf16(p[4], p[5]),
                       pack_bf16(p[6], p[7]));
          if constexpr (PRECISE) {
            float q[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) q[e] = p[e] - bf16_round(p[e]);
            st_shared_v4(sbase + Lay::kPloOff + sb * Lay::kTile + half * Lay::kHalf + off, pack_bf16(q[0], q[1]),
                         pack_bf16(q[2], q[3]), pack_bf16(q[4], q[5]), pack_bf16(q[6], q[7]));
          }
        }
        tile_sum = (ls[0] + ls[1]) + (ls[2] + ls[3]);
        l_run += tile_sum;
        if (tid == 0 && j < 8) SA_TL(kTlAttn, 20 + j);  // P of tile j written
        fence_proxy_async_smem();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&s_free[sb]);
        mbar_arrive(&p_full[sb]);
      }
      if constexpr (OSK) {
        // the tile's share of each row's running softmax mass over both key
        // halves: half 1 passes its (log2 tile mass, log2 running mass) to
        // half 0, which votes to continue while some row's share is at
        // least osk_tau (a row that has seen no key yet always continues)
        const float lA = (warp_active && tile_sum > 0.f) ? m_ref + __log2f(tile_sum) : -INFINITY;
        const float lB = (warp_active && l_run > 0.f) ? m_ref + __log2f(l_run) : -INFINITY;
        if (half == 1) {
          if (j >= 1 && !warp_wait(osk_xfree, (j - 1) & 1)) { failed = true; break; }
          __syncwarp();
          osk_x[r_loc] = make_float2(lA, lB);
          __syncwarp();
          if (lane == 0) mbar_arrive(osk_xfull);
        } else {
          if (!warp_wait(osk_xfull, j & 1)) { failed = true; break; }
          __syncwarp();
          const float2 o = osk_x[r_loc];
          __syncwarp();
          if (lane == 0) mbar_arrive(osk_xfree);
          bool cont = false;
          if (warp_active && me.valid) {
            const float mm = fmaxf(lB, o.y);
            if (mm == -INFINITY) {
              cont = true;
            } else {
              const float num = ex2_approx(lA - mm) + ex2_approx(o.x - mm);
              const float den = ex2_approx(lB - mm) + ex2_approx(o.y - mm);
              cont = !(num < a.osk_tau * den);
            }
          }
          const bool any = __any_sync(0xffffffffu, cont);
          if (lane == 0) {
            osk_vote[(j % kSlots) * 4 + (warp & 3)] = ((uint32_t)j << 1) | (any ? 1u : 0u);
            mbar_arrive(&osk_dec[j % kSlots]);
          }
        }
      }
    }
    if (failed) {
      if (lane == 0) report(a.status, kErrTimeout, kKernAttn, u, 2, warp);
    } else if (warp_active) {
      if (n_run > 0 && !warp_wait(&o_done[(n_run - 1) & 3], ((n_run - 1) >> 2) & 1)) {
        if (lane == 0) report(a.status, kErrTimeout, kKernAttn, u, 3, warp);
      } else {
        have_o = true;
      }
    }
  }

  // ======================= output: all threads =======================
  tc_fence_before();
  __syncthreads();  // every MMA has completed (o_done) and no stage is in use
  if (tid == 0) SA_TL(kTlAttn, 30);
  tc_fence_after();
  if (a.n_split > 1) {
    // this CTA's stages are free for its peers' slices: arm the receive
    // barrier and arrive; the wait comes after the half merge below
    if (tid == 0)
      mbar_arrive_expect_tx(recv_bar, (uint32_t)(a.n_split - 1) * (128u * (16u * (32 / a.n_split) + 8u)));
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  }
  // the two key halves of each row: (m, l) of both, merged per row
  float2* mlx = reinterpret_cast<float2*>(smem + Lay::kStageOff + kMlxOff);  // [2][128]
  if (warp < kSoftWarps)
    mlx[half * 128 + r_loc] = (warp_active && have_o && me.valid) ? make_float2(m_ref, l_run)
                                                                 : make_float2(-INFINITY, 0.f);
  __syncthreads();
  float f0 = 0.f, f1 = 0.f, l_row = 0.f, m_row = -INFINITY;
  if (warp < kSoftWarps) {
    const float2 h0 = mlx[r_loc], h1 = mlx[128 + r_loc];
    m_row = fmaxf(h0.x, h1.x);
    if (m_row != -INFINITY) {
      f0 = ex2_approx(h0.x - m_row);
      f1 = ex2_approx(h1.x - m_row);
      l_row = f0 * h0.y + f1 * h1.y;
    }
  }
  // this thread's 64 output columns of the row: f0 O0 + f1 O1 (unnormalised)
  auto row_out = [&](int c2, float* f) {  // columns 64*half + 32*c2 .. +31
    uint32_t o0[32], o1[32];
    tmem_ld32(tmem + 256 + lane_base + 64 * half + 32 * c2, o0);
    tmem_ld32(tmem + 384 + lane_base + 64 * half + 32 * c2, o1);
    tmem_wait_ld();
#pragma unroll
    for (int e = 0; e < 32; ++e) f[e] = f0 * __uint_as_float(o0[e]) + f1 * __uint_as_float(o1[e]);
  };
  if (a.n_split == 1) {
    if (warp_active && have_o) {
      // partial output: the rows as they are, with (m, l) beside them
      const float inv = a.ml != nullptr ? 1.f : (l_row > 0.f ? 1.f / l_row : 0.f);
      if (a.ml != nullptr && half == 0 && me.valid) a.ml[me.qoff / kD] = make_float2(m_row, l_row);
#pragma unroll 1
      for (int c2 = 0; c2 < 2; ++c2) {
        float f[32];
        if (n_run > 0) {
          row_out(c2, f);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) f[e] = 0.f;
        }
#pragma unroll
        for (int e = 0; e < 32; ++e) f[e] *= inv;
        if (me.valid) store_out(a, me.qoff + 64 * half + 32 * c2, f, 32);
      }
    }
  } else {
    // Key splits of this row tile form one cluster.  Output slice t (128 /
    // n_split columns) is merged by CTA t: every CTA stages, per slice, its
    // unnormalised rows and (m, l) in its own shared memory, then one bulk
    // copy per peer moves the slice into that peer's receive slot, completion
    // counted in bytes on the peer's mbarrier.
    const int ns = a.n_split;
    const int rank = (int)cluster_rank();
    const int cw = 32 / ns;                        // 16-byte chunks per slice row
    // chunk c of row r sits at chunk c ^ swz(r): one row per lane would
    // otherwise put all 32 lanes' 16-byte accesses in the same banks
    const int swz = r_loc & (cw >= 8 ? 7 : cw - 1);
    const uint32_t slot_bytes = 128u * (16u * cw + 8u);  // [128][cw] chunks + [128] (m, l)
    const uint32_t recv = sbase + Lay::kStageOff;                      // [ns] slots, slot s from CTA s
    const uint32_t send = recv + ((ns * slot_bytes + 1023u) & ~1023u);  // [ns] slots, slot t for CTA t
    // every CTA is done with its stages and has armed its receive barrier
    if (tid == 0) SA_TL(kTlAttn, 31);
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
    if (tid == 0) SA_TL(kTlAttn, 32);
    if (warp_active) {
      const bool live = have_o && me.valid;
      if (half == 0)
        for (int t = 0; t < ns; ++t)
          *reinterpret_cast<float2*>(smem + (send - sbase) + t * slot_bytes + 128u * 16u * cw + r_loc * 8u) =
              make_float2(live ? m_row : -INFINITY, live ? l_row : 0.f);
#pragma unroll 1
      for (int c2 = 0; c2 < 2; ++c2) {
        float f[32];
        if (have_o && n_run > 0) {  // warp-uniform: TMEM loads are warp-collective
          row_out(c2, f);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) f[e] = 0.f;
        }
        if (!live) {
#pragma unroll
          for (int e = 0; e < 32; ++e) f[e] = 0.f;
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int chunk = 16 * half + 8 * c2 + q;  // 16-byte chunk of the 512-byte row
          const int owner = chunk / cw;
          st_shared_v4(send + owner * slot_bytes + (uint32_t)((r_loc * cw + ((chunk - owner * cw) ^ swz)) * 16),
                       __float_as_uint(f[4 * q]), __float_as_uint(f[4 * q + 1]), __float_as_uint(f[4 * q + 2]),
                       __float_as_uint(f[4 * q + 3]));
        }
      }
    }
    fence_proxy_async_smem();  // the staged slices are read by the bulk copies (async proxy)
    __syncthreads();
    if (warp == kMmaWarp && lane < ns && lane != rank)
      bulk_copy_to_peer(recv + rank * slot_bytes, send + lane * slot_bytes, slot_bytes, recv_bar, lane);
    bool got = true;
    if (tid == 0) SA_TL(kTlAttn, 33);
    if (warp < kSoftWarps) got = warp_wait(recv_bar, 0);
    if (tid == 0) SA_TL(kTlAttn, 34);
    if (!got && lane == 0) report(a.status, kErrTimeout, kKernAttn, u, 4, warp);
    // all that was sent to this CTA has landed; its own send slots are still
    // read by its peers' copies until every CTA of the cluster arrives here
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
    if (warp_active && me.valid && got) {
      const uint8_t* base = smem + (recv - sbase);
      const uint8_t* own = smem + (send - sbase) + rank * slot_bytes;
      float M = -INFINITY;
      float2 mls[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        if (t < ns) {
          const uint8_t* sl = (t == rank ? own : base + t * slot_bytes);
          mls[t] = *reinterpret_cast<const float2*>(sl + 128u * 16u * cw + r_loc * 8u);
          M = fmaxf(M, mls[t].x);
        }
      }
      float wt[8], L = 0.f;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        wt[t] = 0.f;
        if (t < ns && M != -INFINITY) {
          wt[t] = ex2_approx(mls[t].x - M);
          L += wt[t] * mls[t].y;
        }
      }
      const float inv = a.ml != nullptr ? 1.f : (L > 0.f ? 1.f / L : 0.f);
      if (a.ml != nullptr && rank == 0 && half == 0) a.ml[me.qoff / kD] = make_float2(M, L);
      // the slice's chunks, split between the row's two threads
      const int per = cw / 2 > 0 ? cw / 2 : 1;
      for (int ci = half * per; ci < (half + 1) * per && ci < cw; ++ci) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          if (t >= ns) break;
          const uint32_t sl = (t == rank ? send + rank * slot_bytes : recv + t * slot_bytes);
          const float4 v = ld_shared_f4(sl + (uint32_t)((r_loc * cw + (ci ^ swz)) * 16));
          acc.x += wt[t] * v.x;
          acc.y += wt[t] * v.y;
          acc.z += wt[t] * v.z;
          acc.w += wt[t] * v.w;
        }
        const float f[4] = {acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv};
        store_out(a, me.qoff + (rank * cw + ci) * 4, f, 4);
      }
    }
    if (tid == 0) SA_TL(kTlAttn, 35);
    // every bulk copy out of this CTA has been consumed before it exits
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
  }

  if constexpr (OSK) {
    if (tid == 0 && a.osk_steps != nullptr) a.osk_steps[u] = n_run;
  }
  tc_fence_before();
  __syncthreads();
  if (tid == 0) SA_TL(kTlAttn, 36);
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

int attn_num_units(const AttnArgs& a) {
  const int n_bg = a.prefill ? a.Hkv : a.B * a.Hkv;
  return n_bg * a.n_mtiles * a.n_split;
}

cudaError_t launch_sparse_attn(const AttnArgs& a, const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                               const CUtensorMap& tm_v, bool precise_p, cudaStream_t stream) {
  const int units = attn_num_units(a);
  if (units == 0) return cudaSuccess;
  if (a.n_split != 1 && a.n_split != 2 && a.n_split != 4 && a.n_split != 8) return cudaErrorInvalidValue;
  const bool osk = a.osk_order != nullptr;
  if (osk && (!a.prefill || a.n_split != 1)) return cudaErrorInvalidValue;
  auto kern = osk ? (precise_p ? sparse_attn_kernel<true, true> : sparse_attn_kernel<false, true>)
                  : (precise_p ? sparse_attn_kernel<true, false> : sparse_attn_kernel<false, false>);
  const size_t smem = osk ? (precise_p ? AttnLayout<true>::kSmemOsk : AttnLayout<false>::kSmemOsk)
                          : (precise_p ? AttnLayout<true>::kSmem : AttnLayout<false>::kSmem);
  cudaError_t e = ensure_smem(kern, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(units);
  cfg.blockDim = dim3(kAttnThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = a.n_split;  // the key splits of one row tile share a cluster
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1] = pdl_attribute();
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, kern, a, tm_q, tm_k, tm_v);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace sa

SA_TL_SETTER(sa_timeline_set_attn)
