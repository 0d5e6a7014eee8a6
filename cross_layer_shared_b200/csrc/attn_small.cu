// Sparse decode attention for few query rows per (sequence, KV head):
// R = L_g * G <= 8, as in the per-layer decode mode (one layer, G query heads
// per KV head).  Same definition as attn.cu [IndexCache technical summary
// section 1: attention over the k selected tokens only]:
//   o[r] = sum_t softmax_t(q_r . K_t * scale) V_t  over the valid entries of idx[b]
// The tcgen05 tile of attn.cu is at least 64 rows (128 there): at R = 4 it is
// 97 % padding, and its fixed chain (TMEM, whole-tile gathers, the cluster
// merge of 64 KB slices) sets the launch time.  Here the warp-level
// m16n8k16 MMA fits the shape: 16 rows, of which R are real, computed from
// registers with no allocation or commit chain.
//
// One CTA per (sequence b, KV head g, slice of the k index entries), 4 warps.
// The slices are independent CTAs (no cluster: a cluster must be placed in
// one GPC, and clusters launched while the previous kernel still holds SMs
// were left waiting for room, doubling the launch).  A warp takes 16
// entries at a time, in the transposed products, so that every accumulator
// register holds a real value (lane (gq, tq) = (lane / 4, lane % 4) in the MMA
// layouts):
//   * S^T = K Q^T: the 16 keys on M, the R <= 8 rows on N, 8 k-steps of 16
//     dims.  The dims of a k-step are permuted (the dot product does not care)
//     so that lane tq's operands for k-steps 2i and 2i+1 are the 8 contiguous
//     dims 32i + 8tq.., one 16-byte load per key straight from the cache (the
//     four lanes of a key read 64 contiguous bytes); the query's fragments use
//     the same permutation and are built once;
//   * the 16 V rows go to shared memory by cp.async one pass ahead (a padding
//     entry stages row 0, whose weight is zero), and come back as MMA operands of
//     O^T = V^T P^T by ldmatrix.trans (rows padded to 272 bytes: no bank
//     conflicts);
//   * online softmax: lane (gq, tq) holds rows 2tq, 2tq+1 at keys gq, gq+8;
//     three shuffles reduce a row over the pass.  P^T's fragments want row gq
//     at keys 2tq.. instead, so eight shuffles transpose the weights;
//   * P is split into two bf16 parts (hi + lo: about 16 bits of the fp32
//     weight), so the result carries fp32-level accuracy;
//   * the K and V loads and the entries of the next pass are in flight while
//     a pass computes.
// The 4 warps' (m, l, o) merge in shared memory; each slice writes its
// (m, l, o) to the workspace and counts itself done on a per-(b, g) counter in
// the workspace's zero-once header; the slice that finds itself last merges
// all slices, normalises and stores the rows, and puts the counter back to
// zero.  Softmax references are lazy: a row's reference logit m only moves
// when the running max passes it by more than 8 (log2 units, detected by a
// warp vote), so the weights stay below 2^8 and the accumulators are
// rescaled only then; row sums stay per lane until the end.  Entries < 0
// are padding; entries >= seq_len[b] are reported and skipped.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "attn.cuh"
#include "attn_warp.cuh"
#include "sm100.cuh"
#include "status.cuh"
#include "timeline.cuh"

namespace sa {
namespace {
using namespace wm;

constexpr int kD = 128;
constexpr int kWarpsS = 4;
constexpr int kThreadsS = kWarpsS * 32;
constexpr int kKeysW = 16;                    // entries per warp per pass
constexpr int kSliceKeys = kWarpsS * kKeysW;  // entries per CTA per pass
constexpr int kMaxSplitS = kSmallMaxSplits;
constexpr int kVRow = kD + 8;                 // staged V row: 272 bytes
static_assert(kSmallMaxRows * 16 <= kThreadsS && kMaxSplitS <= 16, "row weights: 16 threads per row");
constexpr size_t kSmemTwoPerSm = 80 * 1024;   // above a third of the SM's shared memory

template <int R>
struct SmallSmem {
  union {
    uint16_t v[2][kWarpsS][kKeysW][kVRow];  // two stages of a warp's 16 V rows
    float wo[kWarpsS][R][kD + 4];        // after the loop: each warp's o
    float pm[kMaxSplitS][R][kD];         // the merging CTA: every slice's o
  };
  uint4 qb[32][4];                       // the query's B fragments, per lane
  float2 wml[kWarpsS][R];                // each warp's (m, l)
  int last;                              // this CTA merges the slices
  float2 sml[kMaxSplitS][R];             // the merging CTA: every slice's (m, l)
  float sf[kMaxSplitS][R];               // the warps' or slices' weight per row
  float2 sL[R];                          // .. each row's (max, sum of weights)
  int64_t out_off[R];                    // each row's first element in O
};



template <int R>
__global__ void __launch_bounds__(kThreadsS, 3) sparse_attn_small_kernel(const AttnArgs a) {
  using Smem = SmallSmem<R>;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
  const int ns = a.n_split;
  const int rank = blockIdx.x % ns;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gq = lane >> 2, tq = lane & 3;
  const int bg = blockIdx.x / ns;
  const int b = bg / a.Hkv, g = bg % a.Hkv;
  if (tid == 0) SA_TL(kTlAttnSmall, 0);
#ifdef SA_TIMELINE
  if (tid == 0 && g_sa_timeline != nullptr) {
    uint32_t smid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    g_sa_timeline[((size_t)kTlAttnSmall * kTimelineCtas + blockIdx.x) * kTimelineSlots + 16] = smid + 1;
  }
#endif
  // this CTA's entries: [rank*per, min(k, (rank+1)*per)), kSliceKeys at a time;
  // this warp's passes: entries e_beg + warp*16 + p*kSliceKeys + [0, 16)
  const int per = ((a.k + ns - 1) / ns + kKeysW - 1) / kKeysW * kKeysW;
  const int e_beg = rank * per, e_end = min(a.k, e_beg + per);
  const int e_w = e_beg + warp * kKeysW;
  const int n_slice_pass = e_w < e_end ? (e_end - e_w + kSliceKeys - 1) / kSliceKeys : 0;
  // entry j of pass p in lane j < 16 (-1: padding or past the slice): the
  // load, then the check, so that several loads can be in flight
  auto entry_raw = [&](int p) -> int {
    const int e = e_w + p * kSliceKeys + lane;
    if (lane >= kKeysW || p >= n_slice_pass || e >= e_end) return -1;
    return __ldcg(&a.idx[(int64_t)b * a.k + e]);
  };
  int len = 0, n_pass = 0, t0 = -1, t1 = -1, r1 = -1;
  const uint16_t* Kb = nullptr;
  const uint16_t* Vb = nullptr;
  auto entry_check = [&](int p, int raw) -> int {
    if (raw >= len) {
      report(a.status, kErrDevice, kKernAttn, (int64_t)b * a.k + e_w + p * kSliceKeys + lane, raw, len);
      return -1;
    }
    return raw;
  };
  // the 16 V rows of a pass into shared memory, two rows per instruction
  // (row 0 for padding entries: finite, and their weight is zero)
  auto stage_v = [&](int tt, int stage) {
    const int ch = lane & 15;
#pragma unroll
    for (int i = 0; i < kKeysW / 2; ++i) {
      const int jj = 2 * i + (lane >> 4);
      const int tv = max(__shfl_sync(0xffffffffu, tt, jj), 0);
      cp_async16(&sm.v[stage][warp][jj][ch * 8], Vb + (int64_t)tv * kD + ch * 8, 16u);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  // K fragments of a pass: keys gq (rows gq of A) and 8 + gq (rows gq + 8)
  uint4 kb[2][4];
  auto load_k = [&](int tt) {
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int tk = max(__shfl_sync(0xffffffffu, tt, 8 * nt + gq), 0);
      const uint4* kp = reinterpret_cast<const uint4*>(Kb + (int64_t)tk * kD + 8 * tq);
#pragma unroll
      for (int i = 0; i < 4; ++i) kb[nt][i] = __ldcg(kp + 4 * i);
    }
  };
  // the first two passes' entries, the sequence's place in the cache, and
  // pass 0's K and V loads (pass p computes while pass p+1's loads and pass
  // p+2's entries are in flight)
  auto prologue = [&]() {
    const int r0 = entry_raw(0);
    r1 = entry_raw(1);
    len = __ldcg(&a.seq_len[b]);
    const int64_t kv_base = (__ldcg(&a.seq_off[b]) * a.Hkv + (int64_t)g * len) * kD;
    Kb = a.K + kv_base;
    Vb = a.V + kv_base;
    n_pass = len > 0 ? n_slice_pass : 0;  // none for an empty sequence: padding stages row 0
    t0 = entry_check(0, r0);
    if (n_pass > 0) {
      stage_v(t0, 0);
      load_k(t0);
    }
  };
  // early: the stream's previous kernel writes none of idx, seq_off,
  // seq_len, K and V, and lets this one start only after its own wait, so
  // they are complete: the first loads overlap that kernel's tail
  if (a.early) prologue();
  pdl_wait();     // the previous kernel of the stream is complete
  pdl_trigger();  // after the wait: a following early launch relies on it
  if (tid == 0) SA_TL(kTlAttnSmall, 1);
  if (!a.early) prologue();
  // query row gq (layer gq / G, head g*G + gq % G) as B fragments of Q^T:
  // for k-step 2i + h, b0 = dims 32i + 8tq + 4h + {0, 1}, b1 = .. + {2, 3};
  // rows gq >= R are zero.  Kept in shared memory, read back each pass.
  if (warp == 0) {
    uint4 q4[4] = {};
    if (gq < a.R) {
      const int h = g * a.G + gq % a.G, l = gq / a.G;
      const uint4* qp = reinterpret_cast<const uint4*>(a.Q + (((int64_t)l * a.B + b) * a.Hq + h) * kD + 8 * tq);
#pragma unroll
      for (int i = 0; i < 4; ++i) q4[i] = __ldcg(qp + 4 * i);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) sm.qb[lane][i] = q4[i];
  }
  if (tid < R) {
    const int h = g * a.G + tid % a.G, l = tid / a.G;
    sm.out_off[tid] = (((int64_t)l * a.B + b) * a.Hq + h) * kD;
  }
  __syncthreads();
  if (tid == 0) SA_TL(kTlAttnSmall, 2);
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};  // rows 2tq, 2tq + 1
  float o[8][4];  // O^T: dims 16mt + gq (+8 for [2], [3]) at rows 2tq ([0], [2]) and 2tq + 1
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
  t1 = entry_check(1, r1);
  if (tid == 0) SA_TL(kTlAttnSmall, 3);
  for (int p = 0; p < n_pass; ++p) {
    const uint32_t live = __ballot_sync(0xffffffffu, t0 >= 0);
    // ---- S^T = K Q^T: lane holds keys gq, gq + 8 at rows 2tq, 2tq + 1 ----
    float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 qf = sm.qb[lane][i];
      mma_bf16(sc, kb[0][i].x, kb[1][i].x, kb[0][i].y, kb[1][i].y, qf.x, qf.y);
      mma_bf16(sc, kb[0][i].z, kb[1][i].z, kb[0][i].w, kb[1][i].w, qf.z, qf.w);
    }
    if (tid == 0 && p < 4) SA_TL(kTlAttnSmall, 4 + p);
    // ---- the next pass's loads ----
    const int rn = entry_raw(p + 2);
    if (p + 1 < n_pass) load_k(t1);
    stage_v(t1, (p + 1) & 1);  // padding only (an empty copy) past the last pass
    // ---- online softmax of rows 2tq + e over the pass (log2 units) ----
    float z[4];  // [e] key gq, [2 + e] key gq + 8, row 2tq + e
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      z[e] = (live >> gq) & 1u ? sc[e] * a.scale_log2 : -INFINITY;
      z[2 + e] = (live >> (gq + 8)) & 1u ? sc[2 + e] * a.scale_log2 : -INFINITY;
    }
    // the reference only moves when some key passes it by more than 8 (rare
    // after a row's first pass: a warp vote decides whether the maxima are
    // reduced); row sums stay per lane (this lane's keys) until the end
    bool over = false;
#pragma unroll
    for (int e = 0; e < 2; ++e) over |= fmaxf(z[e], z[2 + e]) > m_run[e] + 8.f;
    if (__any_sync(0xffffffffu, over)) {
      float alpha[2] = {1.f, 1.f};
      bool moved = false;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float mx = fmaxf(z[e], z[2 + e]);
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        if (mx > m_run[e] + 8.f) {  // also when the row has no reference yet
          alpha[e] = m_run[e] == -INFINITY ? 0.f : ex2f(m_run[e] - mx);
          m_run[e] = mx;
          l_run[e] *= alpha[e];
          moved = true;
        }
      }
      if (moved) {  // this lane's rows (lanes of one tq agree)
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          o[mt][0] *= alpha[0];
          o[mt][1] *= alpha[1];
          o[mt][2] *= alpha[0];
          o[mt][3] *= alpha[1];
        }
      }
    }
    float pw[4];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      pw[e] = z[e] == -INFINITY ? 0.f : ex2f(z[e] - m_run[e]);
      pw[2 + e] = z[2 + e] == -INFINITY ? 0.f : ex2f(z[2 + e] - m_run[e]);
      l_run[e] += pw[e] + pw[2 + e];
    }
    // ---- P^T's B fragments: b0 = row gq at keys 2tq, 2tq + 1, b1 = at keys
    // 2tq + 8, 2tq + 9.  Row gq at key j sits in lane 4 (j mod 8) + gq / 2,
    // half gq % 2 of its (rows 2tq', 2tq' + 1) pair.  hi and lo parts. ----
    uint32_t pb[2][2];  // [hi / lo][b0 / b1]
    {
      const uint32_t h01 = pack_bf16(pw[0], pw[1]), h23 = pack_bf16(pw[2], pw[3]);
      const uint32_t l01 = pack_bf16(pw[0] - bf_lo(h01), pw[1] - bf_hi(h01));
      const uint32_t l23 = pack_bf16(pw[2] - bf_lo(h23), pw[3] - bf_hi(h23));
      const int src0 = 8 * tq + (gq >> 1), src1 = src0 + 4;  // keys 2tq (+8) and 2tq + 1 (+9)
      const uint32_t sel = (gq & 1) ? 0x7632u : 0x5410u;
      const uint32_t w[4] = {h01, h23, l01, l23};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t x = __shfl_sync(0xffffffffu, w[q], src0);
        const uint32_t y = __shfl_sync(0xffffffffu, w[q], src1);
        pb[q >> 1][q & 1] = __byte_perm(x, y, sel);
      }
    }
    asm volatile("cp.async.wait_group 1;" ::: "memory");  // this pass's V rows (the next pass's may be in flight)
    __syncwarp();
    // ---- O^T += V^T P^T: ldmatrix.trans gives V^T's A fragments of 16 dims ----
    const int q8 = lane >> 3, r8 = lane & 7;
    const uint32_t vaddr = (uint32_t)__cvta_generic_to_shared(&sm.v[p & 1][warp][8 * (q8 >> 1) + r8][8 * (q8 & 1)]);
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      uint32_t v0, v1, v2, v3;
      asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                   : "=r"(v0), "=r"(v1), "=r"(v2), "=r"(v3)
                   : "r"(vaddr + mt * 32));
      mma_bf16(o[mt], v0, v1, v2, v3, pb[0][0], pb[0][1]);
      mma_bf16(o[mt], v0, v1, v2, v3, pb[1][0], pb[1][1]);
    }
    if (tid == 0 && p < 4) SA_TL(kTlAttnSmall, 8 + p);
    __syncwarp();  // pass p + 2 overwrites these V rows
    t0 = t1;
    t1 = entry_check(p + 2, rn);
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  // the row sums over the 8 lanes that share each row
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    float v = l_run[e];
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    v += __shfl_xor_sync(0xffffffffu, v, 8);
    v += __shfl_xor_sync(0xffffffffu, v, 16);
    l_run[e] = v;
  }
  // ---- the warps' partials into this CTA's (m, l, o) ----
  __syncthreads();  // every warp is done with its V rows (wo shares their space)
  if (tid == 0) SA_TL(kTlAttnSmall, 12);
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int r = 2 * tq + e;
    if (r < R) {
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        sm.wo[warp][r][16 * mt + gq] = o[mt][e];
        sm.wo[warp][r][16 * mt + 8 + gq] = o[mt][2 + e];
      }
      if (gq == 0) sm.wml[warp][r] = make_float2(m_run[e], l_run[e]);
    }
  }
  // per-row weights of n <= 16 partials (m, l) (the warps', then the
  // slices'): thread tid handles partial tid % 16 of row tid / 16, a
  // 16-lane shuffle reduction per row; f[s][r] = 2^(m_s - M_r), L[r] = sum f l
  auto row_weights = [&](const float2* ml_src, int n) {
    const int r = tid >> 4, s2 = tid & 15;
    const bool mine = r < R && s2 < n;
    const float2 ml = mine ? ml_src[s2 * R + r] : make_float2(-INFINITY, 0.f);
    float M = ml.x;
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off, 16));
    const float f = ml.x == -INFINITY ? 0.f : ex2f(ml.x - M);
    float L = f * ml.y;
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off, 16);
    if (mine) sm.sf[s2][r] = f;
    if (r < R && s2 == 0) sm.sL[r] = make_float2(M, L);
  };
  __syncthreads();
  row_weights(&sm.wml[0][0], kWarpsS);
  __syncthreads();
  // ---- this CTA's (m, l, o) per row: the output itself when the keys are
  // not split, else this slice's partial in the workspace ----
  const bool single = ns == 1;
  float* po = a.small_po + ((int64_t)bg * ns + rank) * R * kD;  // [B*Hkv][ns][R][d]
  float2* pml = a.small_pml + ((int64_t)bg * ns + rank) * R;    // [B*Hkv][ns][R]
  auto store_out = [&](int r, int c, float v) {
    const int64_t off = sm.out_off[r] + c;
    if (a.out_f32)
      reinterpret_cast<float*>(a.O)[off] = v;
    else
      reinterpret_cast<uint16_t*>(a.O)[off] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
  };
  for (int i = tid; i < R * kD; i += kThreadsS) {
    const int r = i / kD, c = i % kD;
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < kWarpsS; ++w) acc += sm.sf[w][r] * sm.wo[w][r][c];
    const float2 ML = sm.sL[r];
    if (single) {
      if (r < a.R) store_out(r, c, ML.y > 0.f ? acc / ML.y : 0.f);
    } else {
      po[i] = acc;
      if (c == 0) pml[r] = ML;
    }
  }
  if (single) {
    if (tid == 0) SA_TL(kTlAttnSmall, 15);
    return;
  }
  // ---- count this slice done; the last one merges ----
  __syncthreads();
  if (tid == 0) SA_TL(kTlAttnSmall, 20);
  if (tid == 0) {
    __threadfence();  // this slice's partial before its count
    sm.last = atomicAdd(&a.small_cnt[bg], 1u) == (unsigned)(ns - 1);
  }
  __syncthreads();
  if (tid == 0) SA_TL(kTlAttnSmall, 13);
  if (!sm.last) return;
  __threadfence();  // the other slices' partials after their counts
  if (tid == 0) SA_TL(kTlAttnSmall, 17);
  const float* po0 = a.small_po + (int64_t)bg * ns * R * kD;
  const float2* pml0 = a.small_pml + (int64_t)bg * ns * R;
  // every slice's partial into shared memory in one round trip (cp.async.cg
  // reads L2, where the other slices' writes are), and their (m, l)
  for (int i = tid; i < ns * R * kD / 4; i += kThreadsS) cp_async16(&sm.pm[0][0][0] + 4 * i, po0 + 4 * i, 16u);
  asm volatile("cp.async.commit_group;" ::: "memory");
  for (int i = tid; i < ns * R; i += kThreadsS) sm.sml[i / R][i % R] = __ldcg(&pml0[i]);
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();
  if (tid == 0) SA_TL(kTlAttnSmall, 18);
  row_weights(&sm.sml[0][0], ns);
  __syncthreads();
  if (tid == 0) SA_TL(kTlAttnSmall, 19);
  for (int i = tid; i < R * kD; i += kThreadsS) {
    const int r = i / kD, c = i % kD;
    if (r >= a.R) continue;
    float acc0 = 0.f, acc1 = 0.f;
    int s2 = 0;
    for (; s2 + 1 < ns; s2 += 2) {
      acc0 += sm.sf[s2][r] * sm.pm[s2][r][c];
      acc1 += sm.sf[s2 + 1][r] * sm.pm[s2 + 1][r][c];
    }
    if (s2 < ns) acc0 += sm.sf[s2][r] * sm.pm[s2][r][c];
    const float L = sm.sL[r].y;
    store_out(r, c, L > 0.f ? (acc0 + acc1) / L : 0.f);
  }
  if (tid == 0) {
    a.small_cnt[bg] = 0;  // ready for the next launch on this workspace
    SA_TL(kTlAttnSmall, 15);
  }
}

template <int R>
cudaError_t launch_small(const AttnArgs& a, cudaStream_t stream) {
  const int ns = a.n_split;
  auto kern = sparse_attn_small_kernel<R>;
  // at most two CTAs per SM: more would let a launch that starts while the
  // previous kernel still holds SMs pile three CTAs onto the free SMs
  const size_t smem = sizeof(SmallSmem<R>) > kSmemTwoPerSm ? sizeof(SmallSmem<R>) : kSmemTwoPerSm;
  cudaError_t e = ensure_smem(kern, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(a.B * a.Hkv * ns));
  cfg.blockDim = dim3(kThreadsS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

SA_TL_SETTER(sa_timeline_set_attn_small)

int small_attn_rows(int R) { return R <= 1 ? 1 : R <= 2 ? 2 : R <= 4 ? 4 : 8; }

int small_attn_splits(int units, int k, int sms, int max_counters) {
  if (units < 1) return 1;
  // as many slices as keep at most two CTAs per SM (one launch wave, every
  // SM busy), each slice at least one pass of all four warps
  int s = 2 * sms / units;
  const int full = (k + kSliceKeys - 1) / kSliceKeys;
  if (s > full) s = full;
  if (s > kMaxSplitS) s = kMaxSplitS;
  if (s < 1 || units > max_counters) return 1;
  // slices are whole 16-entry warp passes: no more slices than that leaves
  // every one with work
  const int chunks = (k + kKeysW - 1) / kKeysW;
  const int per = (chunks + s - 1) / s;
  return (chunks + per - 1) / per;
}

size_t small_attn_scratch_bytes(int units, int ns, int R) {
  if (ns <= 1) return 0;
  const size_t n = (size_t)units * ns * small_attn_rows(R);
  return (n * kD * 4 + 255) / 256 * 256 + (n * 8 + 255) / 256 * 256;
}

cudaError_t launch_sparse_attn_small(const AttnArgs& a, cudaStream_t stream) {
  if (a.prefill || a.ml != nullptr || a.idx_count != nullptr || a.R < 1 || a.R > kSmallMaxRows ||
      a.n_split < 1 || a.n_split > kMaxSplitS || (a.n_split > 1 && (!a.small_cnt || !a.small_po || !a.small_pml)))
    return cudaErrorInvalidValue;
  if (a.B * a.Hkv == 0) return cudaSuccess;
  switch (small_attn_rows(a.R)) {
    case 1: return launch_small<1>(a, stream);
    case 2: return launch_small<2>(a, stream);
    case 4: return launch_small<4>(a, stream);
    default: return launch_small<8>(a, stream);
  }
}

}  // namespace sa
