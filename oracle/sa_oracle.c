/*
 * CPU oracle for cross-layer shared sparse attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, the smoke check and the bench's
 * CPU-baseline leg may load this library.  It shares no code, header, table
 * or helper with the CUDA path in cross_layer_shared_b200/csrc.
 *
 * Each function is the plain definition of one step, computed naively in
 * fp64 (inputs are bf16 bit patterns / fp32 values, widened exactly), with
 * loops in the order the definition is written and OpenMP only over
 * independent outputs.  No blocking, fusion or reordering.
 *
 * Pages followed:
 *   [CLSA]   "Le routage partage entre couches accelere l'attention sparse
 *            de 7x sans perte de qualite" (news article on "CLSA: You Only
 *            Index Once"), section "Comment CLSA fonctionne".
 *   [IC]     "IndexCache: Accelerating Sparse Attention via Cross-Layer
 *            Index Reuse", technical summary, sections 1 (Problematique)
 *            and 2 (Methodologie : IndexCache).
 *   [CA]     "CompactAttention: Accelerating Chunked Prefill with
 *            Block-Union KV Selection", technical summary, section
 *            "Methodologie : CompactAttention" (selection step, execution
 *            step).
 *   [CoSA]   "CoSA: Accelerating Long-Context Inference via Proxy-Kernel
 *            Co-Designed Sparse Attention", lay summary (the kernel-aware
 *            proxy's priority list, the ordered-skipping kernel).
 *
 * The pages name the DSA "lightning indexer" but print no formula for its
 * score; the oracle uses the DSA form score_t = sum_j w_j * ReLU(q_j . k_t)
 * with one key vector per token shared by all indexer heads, no 1/sqrt(d)
 * and no softmax.  The score is rounded once to fp32, the precision in
 * which both sides take the top-k decision.
 *
 * Parity pins for every function live in tests/test_oracle_pins.py.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double bf(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/*
 * Indexer score [IC section 1: the lightning indexer scores every previous
 * token for the current query; CLSA section "Comment CLSA fonctionne": the
 * shared indexer layer computes the scores once].
 *
 * For query q (sequence q_seq[q], last visible key q_pos[q]) and each key
 * t in [0, q_pos[q]]:
 *   dot_j   = sum_c qI[q,j,c] * KI[seq_off[q_seq[q]] + t, c]
 *   score_t = sum_j w[q,j] * max(dot_j, 0)
 * written to scores[q*ld + t] as fp32 (+0 when every dot is <= 0).
 * Entries beyond q_pos are not written.
 */
void oracle_index_score(const uint16_t* qI, const float* w, const uint16_t* KI,
                        const int64_t* seq_off, const int32_t* q_seq, const int32_t* q_pos,
                        int Nq, int H_I, int d_I, float* scores, int64_t ld) {
  for (int q = 0; q < Nq; ++q) {
    const int64_t base = seq_off[q_seq[q]];
    const int64_t n = (int64_t)q_pos[q] + 1;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < n; ++t) {
      const uint16_t* k = KI + (base + t) * d_I;
      double s = 0.0;
      for (int j = 0; j < H_I; ++j) {
        const uint16_t* qj = qI + ((int64_t)q * H_I + j) * d_I;
        double dot = 0.0;
        for (int c = 0; c < d_I; ++c) dot += bf(qj[c]) * bf(k[c]);
        const double relu = dot > 0.0 ? dot : 0.0;
        s += (double)w[(int64_t)q * H_I + j] * relu;
      }
      scores[(int64_t)q * ld + t] = (float)s;
    }
  }
}

typedef struct {
  float s;
  int32_t i;
} scored_t;

/* order: score descending, then index ascending (ties go to the lower index) */
static int by_score_then_index(const void* a, const void* b) {
  const scored_t* x = (const scored_t*)a;
  const scored_t* y = (const scored_t*)b;
  if (x->s > y->s) return -1;
  if (x->s < y->s) return 1;
  return (x->i > y->i) - (x->i < y->i);
}

static int by_index(const void* a, const void* b) {
  const int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
  return (x > y) - (x < y);
}

/*
 * Top-k [IC section 1: the indexer keeps the k most relevant tokens;
 * CLSA: the top-k selection runs once and its index is passed on].
 *
 * Row q: sort the n_valid[q] scores by (score desc, index asc), keep the
 * first min(k, n_valid[q]), emit their indices in ascending order, pad the
 * rest of the row with -1.  top_scores (nullable) gets the matching scores
 * (0 for padding).
 */
void oracle_topk(const float* scores, int64_t ld, const int32_t* n_valid, int Nq, int k,
                 int32_t* idx, float* top_scores) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int q = 0; q < Nq; ++q) {
    const int n = n_valid[q];
    scored_t* all = (scored_t*)malloc(sizeof(scored_t) * (size_t)(n > 0 ? n : 1));
    for (int t = 0; t < n; ++t) {
      all[t].s = scores[(int64_t)q * ld + t];
      all[t].i = t;
    }
    qsort(all, (size_t)n, sizeof(scored_t), by_score_then_index);
    const int m = n < k ? n : k;
    int32_t* row = idx + (int64_t)q * k;
    for (int j = 0; j < m; ++j) row[j] = all[j].i;
    qsort(row, (size_t)m, sizeof(int32_t), by_index);
    for (int j = m; j < k; ++j) row[j] = -1;
    if (top_scores) {
      float* ts = top_scores + (int64_t)q * k;
      for (int j = 0; j < m; ++j) ts[j] = scores[(int64_t)q * ld + row[j]];
      for (int j = m; j < k; ++j) ts[j] = 0.0f;
    }
    free(all);
  }
}

/*
 * Softmax attention of one query row over an explicit key list (helper of
 * the two attention definitions below).
 *   z_t = scale * (q . K_t),  o = sum_t exp(z_t - max z) V_t / sum_t exp(z_t - max z)
 * An empty key list gives o = 0.
 */
static void attend_row(const uint16_t* q, const uint16_t* Kb, const uint16_t* Vb, const int64_t* keys,
                       int64_t n, int d, double scale, double* z, double* o) {
  for (int c = 0; c < d; ++c) o[c] = 0.0;
  if (n == 0) return;
  double m = -INFINITY;
  for (int64_t j = 0; j < n; ++j) {
    const uint16_t* kr = Kb + keys[j] * d;
    double dot = 0.0;
    for (int c = 0; c < d; ++c) dot += bf(q[c]) * bf(kr[c]);
    z[j] = scale * dot;
    if (z[j] > m) m = z[j];
  }
  double den = 0.0;
  for (int64_t j = 0; j < n; ++j) {
    const double p = exp(z[j] - m);
    const uint16_t* vr = Vb + keys[j] * d;
    den += p;
    for (int c = 0; c < d; ++c) o[c] += p * bf(vr[c]);
  }
  for (int c = 0; c < d; ++c) o[c] /= den;
}

/*
 * Sparse decode attention for one layer group reading one KV cache
 * [IC section 1: main attention over the k selected tokens, O(Lk);
 *  IC section 2: S layers reuse the index of the nearest upstream F layer;
 *  CLSA "Comment CLSA fonctionne": every cross-decoder layer gets the same
 *  index over the shared KV cache].
 *
 * Q [L,B,Hq,d]; K,V: sequence b at element offset seq_off[b]*Hkv*d, laid
 * out [Hkv, seq_len[b], d]; idx [B,k] (entries < 0 skipped); query head h
 * reads KV head h / (Hq/Hkv).  O [L,B,Hq,d] in fp64.
 */
void oracle_sparse_decode_attn(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                               const int64_t* seq_off, const int32_t* seq_len, const int32_t* idx,
                               int L, int B, int Hq, int Hkv, int d, int k, double scale,
                               double* O) {
  const int G = Hq / Hkv;
  const int64_t rows = (int64_t)L * B * Hq;
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t r = 0; r < rows; ++r) {
    const int h = (int)(r % Hq);
    const int b = (int)((r / Hq) % B);
    const int g = h / G;
    const uint16_t* Kb = K + seq_off[b] * Hkv * d + (int64_t)g * seq_len[b] * d;
    const uint16_t* Vb = V + seq_off[b] * Hkv * d + (int64_t)g * seq_len[b] * d;
    int64_t* keys = (int64_t*)malloc(sizeof(int64_t) * (size_t)(k > 0 ? k : 1));
    double* z = (double*)malloc(sizeof(double) * (size_t)(k > 0 ? k : 1));
    int64_t n = 0;
    for (int j = 0; j < k; ++j) {
      const int32_t t = idx[(int64_t)b * k + j];
      if (t >= 0) keys[n++] = t;
    }
    attend_row(Q + r * d, Kb, Vb, keys, n, d, scale, z, O + r * d);
    free(keys);
    free(z);
  }
}

/*
 * Block union [CA, selection step]: map every selected token t to its KV
 * block t / block, take the union over every query of the chunk (Q-block
 * union) and over the query heads of each KV group (intra-group union; the
 * index is shared by all heads, so every group gets the same set).  The
 * per-group table T_g is the sorted list of distinct blocks, emitted as
 * CSR: kv_indptr[g+1] = kv_indptr[g] + |T_g|, kv_indices holds the blocks.
 * Returns |T_g|.
 */
int oracle_block_union(const int32_t* idx, int Nq, int k, int S, int block, int Hkv,
                       int32_t* kv_indptr, int32_t* kv_indices) {
  const int nb = (S + block - 1) / block;
  unsigned char* mark = (unsigned char*)calloc((size_t)nb, 1);
  for (int64_t q = 0; q < Nq; ++q)
    for (int j = 0; j < k; ++j) {
      const int32_t t = idx[q * k + j];
      if (t >= 0) mark[t / block] = 1;
    }
  int n = 0;
  for (int bl = 0; bl < nb; ++bl) n += mark[bl];
  kv_indptr[0] = 0;
  for (int g = 0; g < Hkv; ++g) {
    int32_t* out = kv_indices + (int64_t)g * n;
    int m = 0;
    for (int bl = 0; bl < nb; ++bl)
      if (mark[bl]) out[m++] = bl;
    kv_indptr[g + 1] = kv_indptr[g] + n;
  }
  free(mark);
  return n;
}

/*
 * Paged causal attention over the union blocks [CA, execution step: the
 * per-group block table is handed to a dense paged attention kernel that
 * reads the selected blocks in place from the KV-head-major cache
 * [B, H_kv, L, D]].
 *
 * Query p (position q_pos[p]) and head h attend, with softmax, to every key
 * t of the blocks in T_{h/(Hq/Hkv)} with t <= q_pos[p] and t < S.
 * Q [Nq,Hq,d]; K,V [Hkv,S,d]; O [Nq,Hq,d] in fp64.
 */
void oracle_paged_prefill_attn(const uint16_t* Q, const int32_t* q_pos, const uint16_t* K,
                               const uint16_t* V, int S, int Nq, int Hq, int Hkv, int d, int block,
                               const int32_t* kv_indptr, const int32_t* kv_indices, double scale,
                               double* O) {
  const int G = Hq / Hkv;
  const int64_t rows = (int64_t)Nq * Hq;
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t r = 0; r < rows; ++r) {
    const int p = (int)(r / Hq);
    const int h = (int)(r % Hq);
    const int g = h / G;
    const int64_t nblk = kv_indptr[g + 1] - kv_indptr[g];
    int64_t* keys = (int64_t*)malloc(sizeof(int64_t) * (size_t)(nblk * block + 1));
    double* z = (double*)malloc(sizeof(double) * (size_t)(nblk * block + 1));
    int64_t n = 0;
    for (int64_t i = 0; i < nblk; ++i) {
      const int64_t b0 = (int64_t)kv_indices[kv_indptr[g] + i] * block;
      for (int64_t t = b0; t < b0 + block; ++t)
        if (t <= q_pos[p] && t < S) keys[n++] = t;
    }
    attend_row(Q + r * d, K + (int64_t)g * S * d, V + (int64_t)g * S * d, keys, n, d, scale, z,
               O + r * d);
    free(keys);
    free(z);
  }
}

/*
 * The CLSA indexer layer read as a full attention layer whose attention
 * weights give the routing index [CLSA, section "La precision reste
 * stable": the index is computed once from the attention scores of the
 * indexer layer, which sees the same query state and cache as every other
 * layer].  For sequence b and query head h (KV head g = h / (Hq/Hkv)), over
 * every cached token t < seq_len[b]:
 *   z_t     = scale * (Q[b,h] . K[g,t])
 *   p_{h,t} = exp(z_t - max z) / sum_u exp(z_u - max z)     (the attention weights)
 *   O[b,h]  = sum_t p_{h,t} V[g,t]                           (the layer's dense output)
 *   route[b,t] = sum_h p_{h,t}, heads in ascending order, rounded once to fp32
 * Q [B,Hq,d]; K, V as in oracle_sparse_decode_attn; O [B,Hq,d] fp64;
 * route [B, ld] fp32, entries t >= seq_len[b] untouched.  P is scratch of
 * B*Hq*S_max doubles (the weights of every head, summed in head order).
 */
void oracle_indexer_layer_attn(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                               const int64_t* seq_off, const int32_t* seq_len, int B, int Hq, int Hkv,
                               int d, int S_max, double scale, double* O, float* route, int64_t ld,
                               double* P) {
  const int G = Hq / Hkv;
  const int64_t rows = (int64_t)B * Hq;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < rows; ++r) {
    const int b = (int)(r / Hq);
    const int h = (int)(r % Hq);
    const int g = h / G;
    const int64_t S = seq_len[b];
    const uint16_t* Kb = K + seq_off[b] * Hkv * d + (int64_t)g * S * d;
    const uint16_t* Vb = V + seq_off[b] * Hkv * d + (int64_t)g * S * d;
    const uint16_t* q = Q + r * d;
    double* o = O + r * d;
    double* p = P + r * (int64_t)S_max;
    for (int c = 0; c < d; ++c) o[c] = 0.0;
    double m = -INFINITY;
    for (int64_t t = 0; t < S; ++t) {
      double dot = 0.0;
      for (int c = 0; c < d; ++c) dot += bf(q[c]) * bf(Kb[t * d + c]);
      p[t] = scale * dot;
      if (p[t] > m) m = p[t];
    }
    double den = 0.0;
    for (int64_t t = 0; t < S; ++t) den += exp(p[t] - m);
    for (int64_t t = 0; t < S; ++t) {
      p[t] = exp(p[t] - m) / den;
      for (int c = 0; c < d; ++c) o[c] += p[t] * bf(Vb[t * d + c]);
    }
  }
#pragma omp parallel for schedule(static)
  for (int b = 0; b < B; ++b)
    for (int64_t t = 0; t < seq_len[b]; ++t) {
      double acc = 0.0;
      for (int h = 0; h < Hq; ++h) acc += P[((int64_t)b * Hq + h) * S_max + t];
      route[(int64_t)b * ld + t] = (float)acc;
    }
}

/*
 * Context-parallel decode, one rank's attention share [CLSA, "Ce que cela
 * signifie pour l'inference sur longs contextes": contexts past one GPU's
 * reach are left open; sharding each sequence over ranks is this build's
 * reading].  The rows of oracle_sparse_decode_attn, before the division:
 *   m = max_t z_t / ln 2                 (the row's max logit in log2 units)
 *   l = sum_t exp(z_t - max z)           (= sum_t 2^(z_t / ln 2 - m))
 *   o = sum_t exp(z_t - max z) V_t
 * ml holds (m, l) per row; a row with no valid index gets m = -inf, l = 0,
 * o = 0.
 */
void oracle_sparse_decode_attn_partial(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                                       const int64_t* seq_off, const int32_t* seq_len, const int32_t* idx,
                                       int L, int B, int Hq, int Hkv, int d, int k, double scale,
                                       double* O_part, double* ml) {
  const int G = Hq / Hkv;
  const int64_t rows = (int64_t)L * B * Hq;
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t r = 0; r < rows; ++r) {
    const int h = (int)(r % Hq);
    const int b = (int)((r / Hq) % B);
    /* query head h reads KV head h / G of sequence b */
    const int64_t base = (seq_off[b] * Hkv + (int64_t)(h / G) * seq_len[b]) * d;
    const uint16_t* Kb = K + base;
    const uint16_t* Vb = V + base;
    double* o = O_part + r * d;
    for (int c = 0; c < d; ++c) o[c] = 0.0;
    double* z = (double*)malloc(sizeof(double) * (size_t)(k > 0 ? k : 1));
    double mz = -INFINITY;
    for (int j = 0; j < k; ++j) {
      const int32_t t = idx[(int64_t)b * k + j];
      if (t < 0) continue;
      double dot = 0.0;
      for (int c = 0; c < d; ++c) dot += bf(Q[r * d + c]) * bf(Kb[(int64_t)t * d + c]);
      z[j] = dot * scale;
      if (z[j] > mz) mz = z[j];
    }
    double l = 0.0;
    for (int j = 0; j < k; ++j) {
      const int32_t t = idx[(int64_t)b * k + j];
      if (t < 0) continue;
      const double p = exp(z[j] - mz);
      l += p;
      for (int c = 0; c < d; ++c) o[c] += p * bf(Vb[(int64_t)t * d + c]);
    }
    ml[2 * r] = l > 0.0 ? mz / log(2.0) : -INFINITY;
    ml[2 * r + 1] = l;
    free(z);
  }
}

/*
 * The log-sum-exp merge of P partial results of the same rows: with M the
 * largest m_p over parts whose l_p > 0,
 *   O[row] = sum_p 2^(m_p - M) o_p[row] / sum_p 2^(m_p - M) l_p,
 * and O = 0 where every l_p = 0.  O_part [P, rows, d], ml [P, rows, 2].
 */
void oracle_combine_partials(const double* O_part, const double* ml, int P, int64_t rows, int d, double* O) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    double M = -INFINITY;
    for (int p = 0; p < P; ++p)
      if (ml[2 * ((int64_t)p * rows + r) + 1] > 0.0 && ml[2 * ((int64_t)p * rows + r)] > M)
        M = ml[2 * ((int64_t)p * rows + r)];
    double* o = O + r * d;
    for (int c = 0; c < d; ++c) o[c] = 0.0;
    if (M == -INFINITY) continue;
    double den = 0.0;
    for (int p = 0; p < P; ++p) {
      const double m = ml[2 * ((int64_t)p * rows + r)], l = ml[2 * ((int64_t)p * rows + r) + 1];
      if (!(l > 0.0)) continue;
      const double wgt = pow(2.0, m - M);
      den += wgt * l;
      for (int c = 0; c < d; ++c) o[c] += wgt * O_part[((int64_t)p * rows + r) * d + c];
    }
    for (int c = 0; c < d; ++c) o[c] /= den;
  }
}

/*
 * Context-parallel selection: the global top-k of the ranks' candidates.
 * cand_scores / cand_idx [N, B, k] hold every rank's top-k over its own
 * slice (idx < 0 = padding).  Per sequence b: the N*k candidates in order
 * (rank-major, then the rank's order), padding scoring -inf, go through
 * oracle_topk; the positions kept that belong to `rank` become its local
 * indices, in ascending order, then -1.
 */
void oracle_cp_select(const float* cand_scores, const int32_t* cand_idx, int N, int B, int k, int rank,
                      int32_t* local_idx) {
  const int64_t n = (int64_t)N * k;
  float* rows = (float*)malloc(sizeof(float) * (size_t)(B * n > 0 ? B * n : 1));
  int32_t* n_valid = (int32_t*)malloc(sizeof(int32_t) * (size_t)(B > 0 ? B : 1));
  int32_t* sel = (int32_t*)malloc(sizeof(int32_t) * (size_t)(B * k > 0 ? B * k : 1));
  for (int b = 0; b < B; ++b) {
    n_valid[b] = (int32_t)n;
    for (int r = 0; r < N; ++r)
      for (int j = 0; j < k; ++j) {
        const int64_t c = ((int64_t)r * B + b) * k + j;
        rows[(int64_t)b * n + (int64_t)r * k + j] = cand_idx[c] >= 0 ? cand_scores[c] : -INFINITY;
      }
  }
  oracle_topk(rows, n, n_valid, B, k, sel, NULL);
  for (int b = 0; b < B; ++b) {
    int m = 0;
    for (int j = 0; j < k; ++j) {
      const int32_t pos = sel[(int64_t)b * k + j];
      if (pos >= 0 && pos / k == rank) {
        const int32_t t = cand_idx[((int64_t)rank * B + b) * k + pos % k];
        if (t >= 0) local_idx[(int64_t)b * k + m++] = t;
      }
    }
    for (int j = m; j < k; ++j) local_idx[(int64_t)b * k + j] = -1;
  }
  free(rows);
  free(n_valid);
  free(sel);
}

/*
 * Dynamic k [CLSA news article, sections "Le cout : limites de
 * compatibilite" and "Ce que cela signifie pour l'inference sur longs
 * contextes": the indexer layer could set k per query instead of a fixed k;
 * the pages leave the rule open].  Reading: the routing mass.  Row q keeps
 * the smallest number m of its tokens, taken in the top-k order (score
 * descending, lower index first), whose summed score reaches the fraction
 * tau of the row's total score (the sum over all n_valid[q] tokens), but at
 * most k_max; a row that never reaches it keeps min(n, k_max).  Sums are
 * fp64, the total in index order, the running sum in the top-k order.
 * idx[q] gets the m indices ascending, then -1 up to k_max; counts[q] = m.
 */
void oracle_topk_dynamic(const float* scores, int64_t ld, const int32_t* n_valid, int Nq, int k_max, double tau,
                         int32_t* idx, int32_t* counts) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int q = 0; q < Nq; ++q) {
    const int n = n_valid[q];
    double total = 0.0;
    for (int t = 0; t < n; ++t) total += (double)scores[(int64_t)q * ld + t];
    scored_t* all = (scored_t*)malloc(sizeof(scored_t) * (size_t)(n > 0 ? n : 1));
    for (int t = 0; t < n; ++t) {
      all[t].s = scores[(int64_t)q * ld + t];
      all[t].i = t;
    }
    qsort(all, (size_t)n, sizeof(scored_t), by_score_then_index);
    const double target = tau * total;
    int m = n;
    double run = 0.0;
    for (int j = 0; j < n; ++j) {
      run += (double)all[j].s;
      if (run >= target) {
        m = j + 1;
        break;
      }
    }
    if (m > k_max) m = k_max;
    int32_t* row = idx + (int64_t)q * k_max;
    for (int j = 0; j < m; ++j) row[j] = all[j].i;
    qsort(row, (size_t)m, sizeof(int32_t), by_index);
    for (int j = m; j < k_max; ++j) row[j] = -1;
    counts[q] = m;
    free(all);
  }
}

/*
 * CoSA's kernel-aware proxy, read as one priority list per query block
 * [CoSA lay summary: the proxy no longer hands the kernel a yes/no list of
 * blocks but a priority list, most important block first].  The pages
 * give no formula for the priority.  The reading used here takes it from
 * the selection the indexer already made: for query block i (queries
 * i*q_block .. i*q_block + q_block - 1, the last block possibly shorter),
 * block B's hit count is the number of entries (p, e) of those queries'
 * index rows with 0 <= idx[p,e] < S and idx[p,e] / block == B.  The list
 * is the union table T (nT distinct block ids) ordered by hit count,
 * larger first, equal counts by ascending block id.
 * idx [Nq, k]; order [ceil(Nq/q_block), ld], row i's first nT entries.
 */
typedef struct {
  int64_t hits;
  int32_t id;
} kap_t;

static int by_hits_then_id(const void* a, const void* b) {
  const kap_t* x = (const kap_t*)a;
  const kap_t* y = (const kap_t*)b;
  if (x->hits != y->hits) return x->hits > y->hits ? -1 : 1;
  return (x->id > y->id) - (x->id < y->id);
}

void oracle_kap_order(const int32_t* idx, int Nq, int k, int S, int block, int q_block,
                      const int32_t* T, int nT, int32_t* order, int64_t ld) {
  const int nb = (S + block - 1) / block;
  const int n_qb = (Nq + q_block - 1) / q_block;
#pragma omp parallel for schedule(dynamic, 1)
  for (int i = 0; i < n_qb; ++i) {
    int64_t* hits = (int64_t*)calloc((size_t)(nb > 0 ? nb : 1), sizeof(int64_t));
    for (int p = i * q_block; p < Nq && p < (i + 1) * q_block; ++p)
      for (int e = 0; e < k; ++e) {
        const int32_t t = idx[(int64_t)p * k + e];
        if (t >= 0 && t < S) hits[t / block] += 1;
      }
    kap_t* list = (kap_t*)malloc(sizeof(kap_t) * (size_t)(nT > 0 ? nT : 1));
    for (int j = 0; j < nT; ++j) {
      list[j].id = T[j];
      list[j].hits = hits[T[j]];
    }
    qsort(list, (size_t)nT, sizeof(kap_t), by_hits_then_id);
    for (int j = 0; j < nT; ++j) order[(int64_t)i * ld + j] = list[j].id;
    free(list);
    free(hits);
  }
}

/*
 * CoSA's ordered-skipping kernel over the union blocks of a prefill chunk
 * [CoSA lay summary: the kernel reads the blocks in the proxy's priority
 * order, so that a progressive score of what matters is built early, and
 * then skips the later blocks with confidence].  The pages give no skip
 * rule.  The reading used here:
 *   unit (i, g): the rows (p, h) of the queries p of query block i and the
 *     G = Hq/Hkv query heads h of KV group g;
 *   step n: the keys of blocks order[i][2n] and order[i][2n+1] (the last
 *     step may hold one block); row (p, h) sees key t when t <= q_pos[p]
 *     and t < S, with logit z = scale * (Q[p,h] . K[g,t]);
 *   after step n, for each row: M = the largest logit the row has seen in
 *     steps 0..n, a = sum over the row's visible keys of step n of
 *     exp(z - M), L = the same sum over steps 0..n; the step's share
 *     is a / L, and +inf for a row that has seen no key yet;
 *   c_n = the largest share over the unit's rows (the progressive score:
 *     the most any row still gained from step n);
 *   the first step n* with c_n < tau ends the unit after step n* + lag
 *     (the steps already in flight finish), so the unit runs
 *     N = min(n_steps, n* + 1 + lag) steps; N = n_steps when no step
 *     qualifies.  n_steps = ceil(nT / 2).
 *   O[p,h] = softmax attention of row (p, h) over its visible keys of
 *   steps 0..N-1.
 * With steps_in given, unit u runs N = steps_in[u] steps (clamped to
 * [0, n_steps]) whatever the rule says: attention over a prefix of the
 * order fixed by the caller.
 * Only the units listed in units[0..n_units) are computed (all of them
 * when units is NULL); unit id u = g * n_qb + i.  steps[u] = N; crit, when
 * given, gets c_n at crit[u * ld_crit + n] for n < n_steps (the running
 * sums are kept in fp64 over the whole list so that every c_n is known).
 * Q [Nq,Hq,d]; K, V [Hkv,S,d]; O [Nq,Hq,d] fp64 (rows of other units
 * untouched).
 */
void oracle_osk_prefill_attn(const uint16_t* Q, const int32_t* q_pos, const uint16_t* K,
                             const uint16_t* V, int S, int Nq, int Hq, int Hkv, int d, int block,
                             const int32_t* order, int64_t ld, int nT, int q_block, double scale,
                             double tau, int lag, const int32_t* units, int n_units,
                             const int32_t* steps_in, double* O, int32_t* steps, double* crit,
                             int64_t ld_crit) {
  const int G = Hq / Hkv;
  const int n_qb = (Nq + q_block - 1) / q_block;
  const int n_steps = (nT + 1) / 2;
  const int n_all = n_qb * Hkv;
  const int nu = units ? n_units : n_all;
  for (int ui = 0; ui < nu; ++ui) {
    const int u = units ? units[ui] : ui;
    const int g = u / n_qb, i = u % n_qb;
    const int p0 = i * q_block;
    const int p1 = (p0 + q_block < Nq) ? p0 + q_block : Nq;
    const int rows = (p1 - p0) * G;
    const int32_t* list = order + (int64_t)i * ld;
    const uint16_t* Kg = K + (int64_t)g * S * d;
    const uint16_t* Vg = V + (int64_t)g * S * d;
    /* share[r * n_steps + n]: row r's a / L after step n */
    double* share = (double*)malloc(sizeof(double) * (size_t)(rows > 0 ? rows : 1) *
                                    (size_t)(n_steps > 0 ? n_steps : 1));
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < rows; ++r) {
      const int p = p0 + r / G;
      const int h = g * G + r % G;
      const uint16_t* q = Q + ((int64_t)p * Hq + h) * d;
      double M = -INFINITY, L = 0.0;
      double* z = (double*)malloc(sizeof(double) * (size_t)(2 * block));
      for (int n = 0; n < n_steps; ++n) {
        int nz = 0;
        for (int b2 = 2 * n; b2 < 2 * n + 2 && b2 < nT; ++b2) {
          const int64_t t0 = (int64_t)list[b2] * block;
          for (int64_t t = t0; t < t0 + block; ++t) {
            if (t > q_pos[p] || t >= S) continue;
            const uint16_t* kr = Kg + t * d;
            double dot = 0.0;
            for (int c = 0; c < d; ++c) dot += bf(q[c]) * bf(kr[c]);
            z[nz++] = scale * dot;
          }
        }
        double m_step = -INFINITY;
        for (int j = 0; j < nz; ++j)
          if (z[j] > m_step) m_step = z[j];
        const double M_new = m_step > M ? m_step : M;
        double a = 0.0;
        for (int j = 0; j < nz; ++j) a += exp(z[j] - M_new);
        if (M_new != -INFINITY) L = (M == -INFINITY ? 0.0 : L * exp(M - M_new)) + a;
        M = M_new;
        share[(int64_t)r * n_steps + n] = L > 0.0 ? a / L : INFINITY;
      }
      free(z);
    }
    int N = n_steps;
    for (int n = 0; n < n_steps; ++n) {
      double c = -INFINITY;
      for (int r = 0; r < rows; ++r) {
        const double s = share[(int64_t)r * n_steps + n];
        if (s > c) c = s;
      }
      if (crit) crit[(int64_t)u * ld_crit + n] = c;
      if (c < tau && N == n_steps) N = (n + 1 + lag < n_steps) ? n + 1 + lag : n_steps;
    }
    if (steps_in) N = steps_in[u] < 0 ? 0 : (steps_in[u] > n_steps ? n_steps : steps_in[u]);
    steps[u] = N;
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < rows; ++r) {
      const int p = p0 + r / G;
      const int h = g * G + r % G;
      const int64_t cap = (int64_t)2 * N * block + 1;
      int64_t* keys = (int64_t*)malloc(sizeof(int64_t) * (size_t)cap);
      double* z = (double*)malloc(sizeof(double) * (size_t)cap);
      int64_t n = 0;
      for (int b2 = 0; b2 < 2 * N && b2 < nT; ++b2) {
        const int64_t t0 = (int64_t)list[b2] * block;
        for (int64_t t = t0; t < t0 + block; ++t)
          if (t <= q_pos[p] && t < S) keys[n++] = t;
      }
      attend_row(Q + ((int64_t)p * Hq + h) * d, Kg, Vg, keys, n, d, scale, z,
                 O + ((int64_t)p * Hq + h) * d);
      free(keys);
      free(z);
    }
    free(share);
  }
}

/* threads OpenMP will use (reported next to CPU timings) */
int oracle_num_threads(void) {
#ifdef _OPENMP
  extern int omp_get_max_threads(void);
  return omp_get_max_threads();
#else
  return 1;
#endif
}
