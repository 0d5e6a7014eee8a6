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
// Per CTA (256 threads, warp-specialised):
//   warps 5-7  gather 128 K rows and 128 V rows per tile with cp.async into
//              128-byte swizzled shared memory, a 3-deep ring (2 in the
//              precise-P variant); completion signalled on an mbarrier;
//   warp 4     owns TMEM (512 columns: S double buffer + O) and issues
//              S = Q K^T (M=128 rows, N=128 keys, K=d=128) and O += P V
//              (V read MN-major), so the next tile's QK^T overlaps this
//              tile's softmax;
//   warps 0-3  one query row per thread: softmax in registers (exp2
//              domain, running max with lazy rescale: O is rescaled only
//              when the max grows by more than 2^8), P in bf16 (or a hi+lo
//              bf16 pair for fp32 outputs) written over the consumed K
//              tile; warps whose rows are all padding skip the work.
//   Key splits write (O, m, l) partials merged by attn_combine_kernel.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "attn.cuh"
#include "sm100.cuh"

namespace sa {
namespace {

constexpr int kD = 128;
constexpr int kKT = 128;  // keys per tile

template <bool PRECISE>
struct AttnLayout {
  static constexpr int kStages = PRECISE ? 2 : 3;
  static constexpr int kHalf = 16384;  // 128 rows x 128 bytes
  static constexpr int kTile = 2 * kHalf;
  static constexpr int kQOff = 0;
  static constexpr int kStageOff = kTile;
  static constexpr int kStageBytes = 2 * kTile;  // K then V
  static constexpr int kPloOff = kStageOff + kStages * kStageBytes;
  static constexpr int kKposOff = kPloOff + (PRECISE ? 2 * kTile : 0);
  static constexpr int kBarOff = kKposOff + kStages * kKT * 4;
  // kv_full[ST] kv_empty[ST] s_full[2] s_free[2] p_full[2] o_done
  static constexpr int kNBar = 2 * kStages + 7;
  static constexpr int kSlotOff = kBarOff + 8 * kNBar;
  static constexpr size_t kSmem = 1024 + kSlotOff + 16;
};

constexpr int kSoftWarps = 4;       // warps 0-3: one query row per thread
constexpr int kMmaWarp = 4;         // warp 4: TMEM owner, one thread issues MMAs
constexpr int kProdWarp0 = 5;       // warps 5-7: cp.async gathers
constexpr int kProdThreads = 96;
constexpr int kAttnThreads = 256;

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const uint32_t l = __bfloat16_as_ushort(__float2bfloat16_rn(lo));
  const uint32_t h = __bfloat16_as_ushort(__float2bfloat16_rn(hi));
  return l | (h << 16);
}

__device__ __forceinline__ float bf16_round(float x) { return __bfloat162float(__float2bfloat16_rn(x)); }

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// arrive on `bar` when every cp.async issued so far by this thread has landed
__device__ __forceinline__ void cp_async_mbar_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// OR-reduction + barrier over the producer threads (named barrier 1)
__device__ __forceinline__ bool producers_sync_or(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, 96, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
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

struct KeySrc {
  const uint16_t* Kb;
  const uint16_t* Vb;
  int len;     // decode: seq_len[b]
  int base;    // prefill: kv_indptr[g]
  int kbeg, kend;
};

// position of list entry jj, or -1 when the entry is padding / invalid
__device__ __forceinline__ int key_at(const AttnArgs& a, const KeySrc& ks, int b, int jj) {
  if (jj >= ks.kend) return -1;
  if (!a.prefill) {
    const int t = a.idx[(int64_t)b * a.k + jj];
    if (t >= ks.len) {
      report(a.status, kErrDevice, kKernAttn, (int64_t)b * a.k + jj, t, ks.len);
      return -1;
    }
    return t < 0 ? -1 : t;
  }
  const int blk = a.kv_indices[ks.base + jj / a.block];
  const int t = blk * a.block + jj % a.block;
  return (blk >= 0 && t < a.S) ? t : -1;
}

template <bool PRECISE>
__global__ void __launch_bounds__(kAttnThreads, 1) sparse_attn_kernel(const AttnArgs a) {
  using Lay = AttnLayout<PRECISE>;
  constexpr int ST = Lay::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  int* kpos = reinterpret_cast<int*>(smem + Lay::kKposOff);
  uint64_t* kv_full = reinterpret_cast<uint64_t*>(smem + Lay::kBarOff);
  uint64_t* kv_empty = kv_full + ST;
  uint64_t* s_full = kv_empty + ST;
  uint64_t* s_free = s_full + 2;
  uint64_t* p_full = s_free + 2;
  uint64_t* o_done = p_full + 2;
  uint32_t* slot = reinterpret_cast<uint32_t*>(smem + Lay::kSlotOff);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int u = blockIdx.x;
  const int split = u % a.n_split;
  const int mt = (u / a.n_split) % a.n_mtiles;
  const int bg = u / (a.n_split * a.n_mtiles);
  const int b = a.prefill ? 0 : bg / a.Hkv;
  const int g = a.prefill ? bg : bg % a.Hkv;

  KeySrc ks;
  int n_keys;
  if (!a.prefill) {
    ks.len = a.seq_len[b];
    const int64_t base = (a.seq_off[b] * a.Hkv + (int64_t)g * ks.len) * kD;
    ks.Kb = a.K + base;
    ks.Vb = a.V + base;
    ks.base = 0;
    n_keys = a.k;
  } else {
    ks.len = a.S;
    ks.base = a.kv_indptr[g];
    n_keys = (a.kv_indptr[g + 1] - ks.base) * a.block;
    ks.Kb = a.K + (int64_t)g * a.S * kD;
    ks.Vb = a.V + (int64_t)g * a.S * kD;
  }
  ks.kbeg = split * a.keys_per_split;
  ks.kend = min(n_keys, ks.kbeg + a.keys_per_split);
  const int nt = ks.kend > ks.kbeg ? (ks.kend - ks.kbeg + kKT - 1) / kKT : 0;

  if (warp == kMmaWarp) tmem_alloc(slot, 512);
  if (tid == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&kv_full[s], 2 * kProdThreads);  // cp.async completions + plain arrivals
      mbar_init(&kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], kSoftWarps);
      mbar_init(&p_full[i], kSoftWarps);
    }
    mbar_init(o_done, 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  const uint32_t tmem_o = tmem + 256;

  if (warp >= kProdWarp0) {
    // ======================= producers: gather K/V rows =======================
    const int pt = tid - kProdWarp0 * 32;
    const int cchunk = pt & 15, crow0 = pt >> 4;  // rows crow0, crow0 + 6, ...
    for (int j = 0; j < nt; ++j) {
      const int s = j % ST;
      bool bad = false;
      if (j >= ST) bad = !mbar_wait(&kv_empty[s], ((j / ST) & 1) ^ 1, kWaitLimitNs);
      for (int r = pt; r < kKT; r += kProdThreads) kpos[s * kKT + r] = bad ? -1 : key_at(a, ks, b, ks.kbeg + j * kKT + r);
      if (producers_sync_or(bad)) {
        if (pt == 0) report(a.status, kErrTimeout, kKernAttn, u, 0, j);
        break;
      }
      if (j == 0) {
#pragma unroll 4
        for (int rr = crow0; rr < 128; rr += 6) {
          const RowMap rm = map_row(a, b, g, mt * 128 + rr);
          const uint32_t dst = sbase + Lay::kQOff + (cchunk >> 3) * Lay::kHalf + sw128_offset(rr, cchunk & 7);
          cp_async_16(dst, rm.valid ? (const void*)(a.Q + rm.qoff + cchunk * 8) : (const void*)a.Q,
                      rm.valid ? 16u : 0u);
        }
      }
      const uint32_t kdst = sbase + Lay::kStageOff + s * Lay::kStageBytes;
      const uint32_t vdst = kdst + Lay::kTile;
#pragma unroll 4
      for (int rr = crow0; rr < 128; rr += 6) {
        const int t = kpos[s * kKT + rr];
        const uint32_t off = (cchunk >> 3) * Lay::kHalf + sw128_offset(rr, cchunk & 7);
        const int64_t e = (int64_t)(t < 0 ? 0 : t) * kD + cchunk * 8;
        const uint32_t nb = t < 0 ? 0u : 16u;
        cp_async_16(kdst + off, ks.Kb + e, nb);
        cp_async_16(vdst + off, ks.Vb + e, nb);
      }
      cp_async_mbar_arrive(&kv_full[s]);
      mbar_arrive(&kv_full[s]);
    }
    cp_async_wait<0>();
  } else if (warp == kMmaWarp) {
    // ======================= MMA issuer =======================
    if (lane == 0) {
      constexpr uint32_t idesc_qk = umma_idesc_bf16(128, 128, false, false);
      constexpr uint32_t idesc_pv = umma_idesc_bf16(128, 128, false, true);
      auto pv = [&](int i) -> bool {
        if (!mbar_wait(&p_full[i & 1], (i >> 1) & 1, kWaitLimitNs)) return false;
        tc_fence_after();
        const uint32_t kst = sbase + Lay::kStageOff + (i % ST) * Lay::kStageBytes;
        const uint32_t vst = kst + Lay::kTile;
#pragma unroll
        for (int k16 = 0; k16 < 8; ++k16) {
          const uint64_t vd = umma_desc_sw128(vst + k16 * 2048, Lay::kHalf, 1024);
          umma_bf16(tmem_o, umma_desc_sw128(kst + (k16 >> 2) * Lay::kHalf + (k16 & 3) * 32, 16, 1024), vd,
                    idesc_pv, (i | k16) != 0);
          if constexpr (PRECISE)
            umma_bf16(tmem_o,
                      umma_desc_sw128(sbase + Lay::kPloOff + (i & 1) * Lay::kTile + (k16 >> 2) * Lay::kHalf +
                                          (k16 & 3) * 32, 16, 1024),
                      vd, idesc_pv, 1);
        }
        umma_commit(&kv_empty[i % ST]);
        umma_commit(o_done);
        return true;
      };
      bool ok = true;
      for (int j = 0; j < nt && ok; ++j) {
        const int s = j % ST, sb = j & 1;
        ok = mbar_wait(&kv_full[s], (j / ST) & 1, kWaitLimitNs) &&
             mbar_wait(&s_free[sb], ((j >> 1) & 1) ^ 1, kWaitLimitNs);
        if (!ok) break;
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
      if (ok && nt >= 1) ok = pv(nt - 1);
      if (!ok) report(a.status, kErrTimeout, kKernAttn, u, 1, 0);
    }
  } else {
    // ======================= softmax rows (warps 0-3) =======================
    const RowMap me = map_row(a, b, g, mt * 128 + tid);
    const bool warp_active = mt * 128 + warp * 32 < a.R;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    float m_ref = -INFINITY, l_run = 0.f;
    bool failed = false;
    for (int j = 0; j < nt; ++j) {
      const int s = j % ST, sb = j & 1;
      if (!mbar_wait(&s_full[sb], (j >> 1) & 1, kWaitLimitNs)) { failed = true; break; }
      tc_fence_after();
      uint32_t sv[kKT];
      if (warp_active) {
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tmem + sb * 128 + lane_base + c * 32, &sv[c * 32]);
        tmem_wait_ld();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[sb]);
      if (warp_active) {
        if (!mbar_wait(&kv_full[s], (j / ST) & 1, kWaitLimitNs) ||
            (j >= 1 && !mbar_wait(o_done, (j - 1) & 1, kWaitLimitNs))) { failed = true; break; }
        const int* kp = kpos + s * kKT;
        float tmax = -INFINITY;
#pragma unroll
        for (int c = 0; c < kKT; ++c) {
          const int t = kp[c];
          const bool vis = me.valid && t >= 0 && t <= me.limit;
          const float x = vis ? __uint_as_float(sv[c]) * a.scale_log2 : -INFINITY;
          sv[c] = __float_as_uint(x);
          tmax = fmaxf(tmax, x);
        }
        float alpha = 1.f;
        bool rescale = false;
        if (j == 0) {
          m_ref = tmax;
        } else if (tmax > m_ref + 8.f) {
          alpha = exp2f(m_ref - tmax);
          m_ref = tmax;
          rescale = true;
        }
        l_run *= alpha;
        if (__any_sync(0xffffffffu, rescale)) {
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t ov[32];
            tmem_ld32(tmem_o + lane_base + c * 32, ov);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
            tmem_st32(tmem_o + lane_base + c * 32, ov);
          }
          tmem_wait_st();
        }
        const float mr = (m_ref == -INFINITY) ? 0.f : m_ref;
        const uint32_t kst = sbase + Lay::kStageOff + s * Lay::kStageBytes;  // P overwrites the used K tile
        float lsum = 0.f;
#pragma unroll
        for (int c16 = 0; c16 < 16; ++c16) {
          float p[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            p[e] = exp2f(__uint_as_float(sv[c16 * 8 + e]) - mr);
            lsum += p[e];
          }
          const uint32_t off = (c16 >> 3) * Lay::kHalf + sw128_offset(tid, c16 & 7);
          st_shared_v4(kst + off, pack_bf16(p[0], p[1]), pack_bf16(p[2], p[3]), pack_bf16(p[4], p[5]),
                       pack_bf16(p[6], p[7]));
          if constexpr (PRECISE) {
            float q[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) q[e] = p[e] - bf16_round(p[e]);
            st_shared_v4(sbase + Lay::kPloOff + sb * Lay::kTile + off, pack_bf16(q[0], q[1]), pack_bf16(q[2], q[3]),
                         pack_bf16(q[4], q[5]), pack_bf16(q[6], q[7]));
          }
        }
        l_run += lsum;
        fence_proxy_async_smem();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[sb]);
    }
    if (failed) {
      if (lane == 0) report(a.status, kErrTimeout, kKernAttn, u, 2, warp);
    } else if (warp_active) {
      if (nt > 0 && !mbar_wait(o_done, (nt - 1) & 1, kWaitLimitNs)) {
        if (lane == 0) report(a.status, kErrTimeout, kKernAttn, u, 3, warp);
      } else {
        tc_fence_after();
        const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
        const int units = gridDim.x;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {  // 32 output columns at a time
          uint32_t ov[32];
          if (nt > 0) {
            tmem_ld32(tmem_o + lane_base + c * 32, ov);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = 0u;
          }
          if (!me.valid) continue;
          if (a.n_split == 1) {
            if (a.out_f32) {
              float4* o = reinterpret_cast<float4*>(reinterpret_cast<float*>(a.O) + me.qoff + c * 32);
#pragma unroll
              for (int e = 0; e < 8; ++e)
                o[e] = make_float4(__uint_as_float(ov[4 * e]) * inv, __uint_as_float(ov[4 * e + 1]) * inv,
                                   __uint_as_float(ov[4 * e + 2]) * inv, __uint_as_float(ov[4 * e + 3]) * inv);
            } else {
              uint4* o = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(a.O) + me.qoff + c * 32);
#pragma unroll
              for (int e = 0; e < 4; ++e)
                o[e] = make_uint4(pack_bf16(__uint_as_float(ov[8 * e]) * inv, __uint_as_float(ov[8 * e + 1]) * inv),
                                  pack_bf16(__uint_as_float(ov[8 * e + 2]) * inv, __uint_as_float(ov[8 * e + 3]) * inv),
                                  pack_bf16(__uint_as_float(ov[8 * e + 4]) * inv, __uint_as_float(ov[8 * e + 5]) * inv),
                                  pack_bf16(__uint_as_float(ov[8 * e + 6]) * inv, __uint_as_float(ov[8 * e + 7]) * inv));
            }
          } else {
            uint4* po = reinterpret_cast<uint4*>(a.part + ((int64_t)u * 128 + tid) * kD + c * 32);
#pragma unroll
            for (int e = 0; e < 8; ++e) po[e] = make_uint4(ov[4 * e], ov[4 * e + 1], ov[4 * e + 2], ov[4 * e + 3]);
          }
        }
        if (me.valid && a.n_split > 1) {
          float2* pml = reinterpret_cast<float2*>(a.part + (int64_t)units * 128 * kD) + (int64_t)u * 128 + tid;
          *pml = make_float2(m_ref, l_run);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Merge the key-split partials of one output row per warp:
//   o = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s,  M = max_s m_s.
__global__ void __launch_bounds__(256) attn_combine_kernel(const AttnArgs a, int units) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int n_bg = a.prefill ? a.Hkv : a.B * a.Hkv;
  if (warp >= n_bg * a.R) return;
  const int bg = warp / a.R, r = warp % a.R;
  const int b = a.prefill ? 0 : bg / a.Hkv;
  const int g = a.prefill ? bg : bg % a.Hkv;
  const int mt = r / 128, lr = r % 128;
  const float2* ml = reinterpret_cast<const float2*>(a.part + (int64_t)units * 128 * kD);
  float M = -INFINITY;
  for (int s = 0; s < a.n_split; ++s) {
    const int uu = (bg * a.n_mtiles + mt) * a.n_split + s;
    M = fmaxf(M, ml[(int64_t)uu * 128 + lr].x);
  }
  const float Mr = (M == -INFINITY) ? 0.f : M;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float lsum = 0.f;
  for (int s = 0; s < a.n_split; ++s) {
    const int uu = (bg * a.n_mtiles + mt) * a.n_split + s;
    const float2 v = ml[(int64_t)uu * 128 + lr];
    const float wgt = exp2f(v.x - Mr);
    lsum += wgt * v.y;
    const float4 o = reinterpret_cast<const float4*>(a.part + ((int64_t)uu * 128 + lr) * kD)[lane];
    acc.x += wgt * o.x;
    acc.y += wgt * o.y;
    acc.z += wgt * o.z;
    acc.w += wgt * o.w;
  }
  const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
  const RowMap rm = map_row(a, b, g, r);
  if (a.out_f32) {
    reinterpret_cast<float4*>(reinterpret_cast<float*>(a.O) + rm.qoff)[lane] =
        make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  } else {
    reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(a.O) + rm.qoff)[lane] =
        make_uint2(pack_bf16(acc.x * inv, acc.y * inv), pack_bf16(acc.z * inv, acc.w * inv));
  }
}

}  // namespace

int attn_num_units(const AttnArgs& a) {
  const int n_bg = a.prefill ? a.Hkv : a.B * a.Hkv;
  return n_bg * a.n_mtiles * a.n_split;
}

size_t attn_partial_bytes(int units) { return (size_t)units * 128 * (kD + 2) * sizeof(float); }

cudaError_t launch_sparse_attn(const AttnArgs& a, bool precise_p, cudaStream_t stream) {
  const int units = attn_num_units(a);
  if (units == 0) return cudaSuccess;
  cudaError_t e;
  if (precise_p) {
    auto kern = sparse_attn_kernel<true>;
    e = ensure_smem(kern, AttnLayout<true>::kSmem);
    if (e != cudaSuccess) return e;
    kern<<<units, kAttnThreads, AttnLayout<true>::kSmem, stream>>>(a);
  } else {
    auto kern = sparse_attn_kernel<false>;
    e = ensure_smem(kern, AttnLayout<false>::kSmem);
    if (e != cudaSuccess) return e;
    kern<<<units, kAttnThreads, AttnLayout<false>::kSmem, stream>>>(a);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess || a.n_split == 1) return e;
  const int n_bg = a.prefill ? a.Hkv : a.B * a.Hkv;
  const int64_t rows = (int64_t)n_bg * a.R;
  const int blocks = (int)((rows * 32 + 255) / 256);
  attn_combine_kernel<<<blocks, 256, 0, stream>>>(a, units);
  return cudaGetLastError();
}

}  // namespace sa
