// Sparse decode attention for 9 to 128 query rows per (sequence, KV head),
// a fused layer group (rows = L_g x G).  Same definition as attn.cu
// [IndexCache technical summary section 1: attention over the k selected
// tokens only; a group's layers share the index]:
//   o[r] = sum_t softmax_t(q_r . K_t * scale) V_t  over the valid entries of idx[b]
//
// The 128-row tcgen05 kernel of attn.cu gathers a whole 128-key tile per
// stage with one CTA per SM and merges its key splits through 64 KB
// distributed-shared-memory slices; its gathers run at about 25 GB/s per SM.
// This kernel keeps more loads in flight with smaller units and runs the
// contractions as warp-level m16n8k16 MMAs:
//   * one CTA per (sequence b, KV head g, slice of the index entries), one
//     warp per 16 query rows (rows 16w .. 16w+15; rows past R are zero);
//   * the CTA reads its slice of the index into shared memory (checked),
//     then walks it 16 entries at a time.  Every thread copies a
//     share of the pass's 16 K rows and 16 V rows into shared memory with
//     cp.async, two passes ahead of the one computing (three stages; rows
//     padded to 272 bytes, so ldmatrix reads them without bank conflicts);
//     a padding entry stages row 0, whose weight is zero;
//   * each warp computes S^T = K Q^T for its 16 rows (keys on M, rows on
//     N: two n-tiles), the online softmax of its rows (lazy reference: it
//     moves only when the running max passes it by more than 8 in log2
//     units, which a warp vote detects; row sums stay per lane until the
//     end), and O^T += V^T P^T with V^T and K from ldmatrix (the K tile
//     and the V tile of a pass are shared by all warps);
//   * P is rounded to bf16 for bf16 outputs (as the tcgen05 kernel does)
//     and split into two bf16 parts (hi + lo) for fp32 outputs.
// With one slice the CTA normalises and stores its rows.  Otherwise each
// slice writes its rows' (m, l, o) to the workspace and a second kernel,
// launched behind it with programmatic dependent launch, merges the slices
// of each (b, g) and 8 rows per CTA.  Entries < 0 are padding; entries >=
// seq_len[b] are reported and skipped.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "attn.cuh"
#include "attn_warp.cuh"
#include "sm100.cuh"
#include "status.cuh"

namespace sa {
namespace {
using namespace wm;

constexpr int kD = 128;
constexpr int kKeysP = 16;                 // entries per pass
constexpr int kStagesM = 3;
constexpr int kVRowM = kD + 8;             // staged row: 272 bytes
constexpr int kMaxWarpsM = kMidMaxRows / 16;
constexpr int kMaxSplitM = kMidMaxSplits;

struct MidSmem {
  uint16_t k[kStagesM][kKeysP][kVRowM];
  uint16_t v[kStagesM][kKeysP][kVRowM];
  int ent[kMidMaxSlice];                   // the slice's checked entries (-1: padding)
};

template <bool kPreciseP>
__global__ void __launch_bounds__(kMaxWarpsM * 32) sparse_attn_mid_kernel(const AttnArgs a) {
  __shared__ MidSmem sm;
  const int ns = a.n_split;
  const int rank = blockIdx.x % ns;
  const int bg = blockIdx.x / ns;
  const int b = bg / a.Hkv, g = bg % a.Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nthreads = blockDim.x;
  const int gq = lane >> 2, tq = lane & 3;
  pdl_wait();     // the index comes from the top-k before this kernel
  pdl_trigger();
  const int len = __ldcg(&a.seq_len[b]);
  const int64_t kv_base = (__ldcg(&a.seq_off[b]) * a.Hkv + (int64_t)g * len) * kD;
  const uint16_t* Kb = a.K + kv_base;
  const uint16_t* Vb = a.V + kv_base;
  // this CTA's entries [e_beg, e_end), in whole passes
  const int per = ((a.k + ns - 1) / ns + kKeysP - 1) / kKeysP * kKeysP;
  const int e_beg = rank * per, e_end = min(a.k, e_beg + per);
  const int n_pass = e_beg < e_end && len > 0 ? (e_end - e_beg + kKeysP - 1) / kKeysP : 0;
  // the slice's entries, checked, into shared memory (one round trip; the
  // passes then issue their copies without waiting on a load)
  for (int i = tid; i < e_end - e_beg; i += nthreads) {
    int t = __ldcg(&a.idx[(int64_t)b * a.k + e_beg + i]);
    if (t >= len) {
      report(a.status, kErrDevice, kKernAttn, (int64_t)b * a.k + e_beg + i, t, len);
      t = -1;
    }
    sm.ent[i] = t;
  }
  for (int i = (e_end > e_beg ? e_end - e_beg : 0) + tid; i < n_pass * kKeysP; i += nthreads) sm.ent[i] = -1;
  __syncthreads();
  // a pass's 16 K and 16 V rows into stage `st`: 512 chunks of 16 bytes
  // (a padding entry stages row 0, whose weight is zero)
  auto issue = [&](int p, int st) {
    if (p < n_pass) {
      for (int c = tid; c < 2 * kKeysP * 16; c += nthreads) {
        const int j = (c >> 4) & (kKeysP - 1), ch = c & 15, kind = c >> 8;
        const int t = sm.ent[p * kKeysP + j];
        const int row = t >= 0 ? t : 0;
        cp_async16(kind ? &sm.v[st][j][ch * 8] : &sm.k[st][j][ch * 8],
                   (kind ? Vb : Kb) + (int64_t)row * kD + ch * 8, 16u);
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  issue(0, 0);
  issue(1, 1);
  // this warp's rows as B fragments of Q^T: n-tile nt holds rows
  // 16w + 8nt + gq; k-step s: b0 = dims 16s + 2tq + {0,1}, b1 = 16s + 8 + 2tq + {0,1}
  uint32_t qb[2][8][2];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    const int r = 16 * warp + 8 * nt + gq;
    const bool real = r < a.R;
    const int h = g * a.G + (real ? r % a.G : 0), l = real ? r / a.G : 0;
    const uint32_t* qp =
        reinterpret_cast<const uint32_t*>(a.Q + (((int64_t)l * a.B + b) * a.Hq + h) * kD + 2 * tq);
#pragma unroll
    for (int s2 = 0; s2 < 8; ++s2) {
      qb[nt][s2][0] = real ? __ldcg(qp + 8 * s2) : 0u;
      qb[nt][s2][1] = real ? __ldcg(qp + 8 * s2 + 4) : 0u;
    }
  }
  float m_run[2][2], l_run[2][2];  // [n-tile][e]: row 16w + 8nt + 2tq + e
  float o[8][2][4];                // O^T: dims 16mt + gq (+8 for [2], [3]); rows 2tq ([0], [2]), 2tq + 1
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    m_run[nt][0] = m_run[nt][1] = -INFINITY;
    l_run[nt][0] = l_run[nt][1] = 0.f;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) o[mt][nt][0] = o[mt][nt][1] = o[mt][nt][2] = o[mt][nt][3] = 0.f;
  }
  const int q8 = lane >> 3, r8 = lane & 7;
  for (int p = 0; p < n_pass; ++p) {
    const int st = p % kStagesM;
    asm volatile("cp.async.wait_group 1;" ::: "memory");  // this thread's copies of pass p
    __syncthreads();  // every thread's copies of pass p; every warp done with pass p - 1
    issue(p + 2, (p + 2) % kStagesM);  // into the stage pass p - 1 used
    const bool live0 = sm.ent[p * kKeysP + gq] >= 0, live1 = sm.ent[p * kKeysP + gq + 8] >= 0;
    // ---- S^T = K Q^T: lane holds keys gq, gq + 8 at rows 2tq, 2tq + 1 of each n-tile ----
    float sc[2][4] = {};
    const uint32_t kaddr =
        (uint32_t)__cvta_generic_to_shared(&sm.k[st][(lane & 7) + 8 * ((lane >> 3) & 1)][8 * (lane >> 4)]);
#pragma unroll
    for (int s2 = 0; s2 < 8; ++s2) {
      uint32_t k0, k1, k2, k3;
      ldsm_x4(kaddr + 32 * s2, k0, k1, k2, k3);
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) mma_bf16(sc[nt], k0, k1, k2, k3, qb[nt][s2][0], qb[nt][s2][1]);
    }
    // ---- online softmax of each row over the pass (log2 units).  The
    // row's reference only moves when some key passes it by more than 8,
    // which after a row's first pass is rare: a warp vote decides whether
    // the row maxima are reduced at all.  Row sums stay per lane (each lane
    // adds its own keys' weights) until the end. ----
    float z[2][4];
    bool over = false;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        z[nt][e] = live0 ? sc[nt][e] * a.scale_log2 : -INFINITY;
        z[nt][2 + e] = live1 ? sc[nt][2 + e] * a.scale_log2 : -INFINITY;
        over |= fmaxf(z[nt][e], z[nt][2 + e]) > m_run[nt][e] + 8.f;
      }
    if (__any_sync(0xffffffffu, over)) {
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        float alpha[2] = {1.f, 1.f};
        bool moved = false;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float mx = fmaxf(z[nt][e], z[nt][2 + e]);
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
          if (mx > m_run[nt][e] + 8.f) {  // also when the row has no reference yet
            alpha[e] = m_run[nt][e] == -INFINITY ? 0.f : ex2f(m_run[nt][e] - mx);
            m_run[nt][e] = mx;
            l_run[nt][e] *= alpha[e];
            moved = true;
          }
        }
        if (moved) {
#pragma unroll
          for (int mt = 0; mt < 8; ++mt) {
            o[mt][nt][0] *= alpha[0];
            o[mt][nt][1] *= alpha[1];
            o[mt][nt][2] *= alpha[0];
            o[mt][nt][3] *= alpha[1];
          }
        }
      }
    }
    float pw[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        pw[nt][e] = z[nt][e] == -INFINITY ? 0.f : ex2f(z[nt][e] - m_run[nt][e]);
        pw[nt][2 + e] = z[nt][2 + e] == -INFINITY ? 0.f : ex2f(z[nt][2 + e] - m_run[nt][e]);
        l_run[nt][e] += pw[nt][e] + pw[nt][2 + e];  // this lane's keys only
      }
    // ---- P^T's B fragments per n-tile: b0 = row gq at keys 2tq, 2tq + 1,
    // b1 = at 2tq + 8, 2tq + 9.  Row gq at key j sits in lane 4 (j mod 8) +
    // gq / 2, half gq % 2 of its (rows 2tq', 2tq' + 1) pair. ----
    uint32_t pb[2][2][2];  // [n-tile][hi / lo][b0 / b1]
    {
      const int src0 = 8 * tq + (gq >> 1), src1 = src0 + 4;
      const uint32_t sel = (gq & 1) ? 0x7632u : 0x5410u;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const uint32_t h01 = pack_bf16(pw[nt][0], pw[nt][1]), h23 = pack_bf16(pw[nt][2], pw[nt][3]);
        pb[nt][0][0] = __byte_perm(__shfl_sync(0xffffffffu, h01, src0), __shfl_sync(0xffffffffu, h01, src1), sel);
        pb[nt][0][1] = __byte_perm(__shfl_sync(0xffffffffu, h23, src0), __shfl_sync(0xffffffffu, h23, src1), sel);
        if (kPreciseP) {
          const uint32_t l01 = pack_bf16(pw[nt][0] - bf_lo(h01), pw[nt][1] - bf_hi(h01));
          const uint32_t l23 = pack_bf16(pw[nt][2] - bf_lo(h23), pw[nt][3] - bf_hi(h23));
          pb[nt][1][0] = __byte_perm(__shfl_sync(0xffffffffu, l01, src0), __shfl_sync(0xffffffffu, l01, src1), sel);
          pb[nt][1][1] = __byte_perm(__shfl_sync(0xffffffffu, l23, src0), __shfl_sync(0xffffffffu, l23, src1), sel);
        }
      }
    }
    // ---- O^T += V^T P^T ----
    const uint32_t vaddr =
        (uint32_t)__cvta_generic_to_shared(&sm.v[st][8 * (q8 >> 1) + r8][8 * (q8 & 1)]);
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      uint32_t v0, v1, v2, v3;
      ldsm_x4_trans(vaddr + mt * 32, v0, v1, v2, v3);
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        mma_bf16(o[mt][nt], v0, v1, v2, v3, pb[nt][0][0], pb[nt][0][1]);
        if (kPreciseP) mma_bf16(o[mt][nt], v0, v1, v2, v3, pb[nt][1][0], pb[nt][1][1]);
      }
    }
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  // the row sums over the 8 lanes that share each row
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float v = l_run[nt][e];
      v += __shfl_xor_sync(0xffffffffu, v, 4);
      v += __shfl_xor_sync(0xffffffffu, v, 8);
      v += __shfl_xor_sync(0xffffffffu, v, 16);
      l_run[nt][e] = v;
    }
  // ---- this warp's rows: the output (one slice) or the slice's partial ----
  const bool single = ns == 1;
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int r = 16 * warp + 8 * nt + 2 * tq + e;
      if (r >= a.R) continue;
      const int h = g * a.G + r % a.G, l = r / a.G;
      const int64_t off = (((int64_t)l * a.B + b) * a.Hq + h) * kD;
      const float L = l_run[nt][e];
      if (single) {
        const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const float v = o[mt][nt][2 * hh + e] * inv;
            const int64_t idx = off + 16 * mt + 8 * hh + gq;
            if (a.out_f32)
              reinterpret_cast<float*>(a.O)[idx] = v;
            else
              reinterpret_cast<uint16_t*>(a.O)[idx] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
          }
        }
      } else {
        float* po = a.small_po + (((int64_t)bg * ns + rank) * a.R + r) * kD;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          po[16 * mt + gq] = o[mt][nt][e];
          po[16 * mt + 8 + gq] = o[mt][nt][2 + e];
        }
        if (gq == 0) a.small_pml[((int64_t)bg * ns + rank) * a.R + r] = make_float2(m_run[nt][e], L);
      }
    }
  }
}

// The merge of a split (b, g)'s slices, 8 rows per CTA (one warp per row,
// lane l on dims 4l .. 4l+3): o = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s.
__global__ void __launch_bounds__(256) sparse_attn_mid_combine(const AttnArgs a) {
  const int ns = a.n_split;
  const int groups = (a.R + 7) / 8;
  const int bg = blockIdx.x / groups, rg = blockIdx.x % groups;
  const int b = bg / a.Hkv, g = bg % a.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = 8 * rg + warp;
  pdl_wait();     // the slices' partials are complete
  pdl_trigger();  // after the wait: a following early launch relies on it
  if (r >= a.R) return;
  float2 ml[kMaxSplitM];
  float M = -INFINITY;
#pragma unroll
  for (int s = 0; s < kMaxSplitM; ++s) {
    ml[s] = s < ns ? __ldcg(&a.small_pml[((int64_t)bg * ns + s) * a.R + r]) : make_float2(-INFINITY, 0.f);
    M = fmaxf(M, ml[s].x);
  }
  float L = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int s = 0; s < kMaxSplitM; ++s) {
    if (s < ns && ml[s].x != -INFINITY) {
      const float f = ex2f(ml[s].x - M);
      L += f * ml[s].y;
      const float4 v = __ldcg(reinterpret_cast<const float4*>(a.small_po + (((int64_t)bg * ns + s) * a.R + r) * kD) +
                              lane);
      acc.x += f * v.x;
      acc.y += f * v.y;
      acc.z += f * v.z;
      acc.w += f * v.w;
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  const int h = g * a.G + r % a.G, l = r / a.G;
  const int64_t off = (((int64_t)l * a.B + b) * a.Hq + h) * kD + 4 * lane;
  if (a.out_f32) {
    reinterpret_cast<float4*>(reinterpret_cast<float*>(a.O) + off)[0] =
        make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  } else {
    const uint32_t lo = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(acc.x * inv)) |
                        ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(acc.y * inv)) << 16);
    const uint32_t hi = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(acc.z * inv)) |
                        ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(acc.w * inv)) << 16);
    reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(a.O) + off)[0] = make_uint2(lo, hi);
  }
}

template <typename Kernel>
cudaError_t launch_pdl_mid(Kernel kern, unsigned grid, unsigned block, const AttnArgs& a, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

int mid_attn_splits(int units, int R, int k, int sms) {
  if (units < 1) return 1;
  const int warps = (R + 15) / 16;
  // about 12 warps per SM in all; whole 16-entry passes for every slice
  int s = 12 * sms / (units * warps);
  const int passes = (k + kKeysP - 1) / kKeysP;
  if (s > passes) s = passes;
  if (s > kMaxSplitM) s = kMaxSplitM;
  // a slice's entries fit the kernel's shared memory
  const int min_s = (k + kMidMaxSlice - 1) / kMidMaxSlice;
  if (s < min_s) s = min_s;
  if (s < 1) return 1;
  const int per = (passes + s - 1) / s;
  return (passes + per - 1) / per;
}

size_t mid_attn_scratch_bytes(int units, int ns, int R) {
  if (ns <= 1) return 0;
  const size_t n = (size_t)units * ns * R;
  return (n * kD * 4 + 255) / 256 * 256 + (n * 8 + 255) / 256 * 256;
}

cudaError_t launch_sparse_attn_mid(const AttnArgs& a, cudaStream_t stream) {
  if (a.prefill || a.ml != nullptr || a.idx_count != nullptr || a.R < 1 || a.R > kMidMaxRows || a.n_split < 1 ||
      a.n_split > kMaxSplitM || (a.n_split > 1 && (!a.small_po || !a.small_pml)))
    return cudaErrorInvalidValue;
  const unsigned units = (unsigned)(a.B * a.Hkv);
  if (units == 0) return cudaSuccess;
  const unsigned warps = (unsigned)((a.R + 15) / 16);
  cudaError_t e = a.out_f32 ? launch_pdl_mid(sparse_attn_mid_kernel<true>, units * a.n_split, warps * 32, a, stream)
                            : launch_pdl_mid(sparse_attn_mid_kernel<false>, units * a.n_split, warps * 32, a, stream);
  if (e != cudaSuccess || a.n_split == 1) return e;
  return launch_pdl_mid(sparse_attn_mid_combine, units * (unsigned)((a.R + 7) / 8), 256, a, stream);
}

}  // namespace sa
