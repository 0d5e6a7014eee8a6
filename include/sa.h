/*
 * libsa - cross-layer shared sparse attention on B200 (sm_100a).
 *
 * C ABI of the hot path: a lightweight indexer scores every cached key
 * against the current query, a top-k over the whole context picks the
 * tokens to attend to, and that one index is shared by a group of layers
 * reading one KV cache, each running softmax attention over only the
 * selected tokens.  A chunked-prefill variant unions the selected KV blocks
 * per GQA group into a block table and attends to those blocks in place.
 *
 * Pages this interface follows (cited per entry below):
 *   [CLSA] "Le routage partage entre couches accelere l'attention sparse de
 *          7x sans perte de qualite" - news article on "CLSA: You Only Index
 *          Once", section "Comment CLSA fonctionne".
 *   [IC]   "IndexCache: Accelerating Sparse Attention via Cross-Layer Index
 *          Reuse" - technical summary, sections 1 "Problematique" and
 *          2 "Methodologie : IndexCache".
 *   [CA]   "CompactAttention: Accelerating Chunked Prefill with Block-Union
 *          KV Selection" - technical summary, section "Methodologie :
 *          CompactAttention" (selection step, execution step).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every tensor pointer is DEVICE memory owned by the caller.  The library
 *   never allocates, frees or synchronises inside a compute call; each call
 *   only enqueues work on `stream` (a cudaStream_t; NULL = legacy default
 *   stream) and returns.
 * - bf16 tensors are passed as `const void*` holding IEEE bfloat16 bit
 *   patterns.  Rows of bf16 tensors must start 16-byte aligned (all the
 *   shapes below have d or d_I a multiple of 64, so a 16-byte aligned base
 *   suffices).
 * - Argument errors are detected on the host before anything is enqueued;
 *   the call then returns SA_ERR_INVALID_ARG / SA_ERR_UNSUPPORTED /
 *   SA_ERR_WORKSPACE and sa_last_error() describes the problem.
 * - Errors only the device can see (an index out of range, a sequence length
 *   above the stated maximum, a bounded wait that gave up) are recorded in
 *   the status block at the start of the workspace and read back with
 *   sa_read_device_status().  The kernel skips the offending element instead
 *   of touching memory outside the buffers.
 * - Workspace: `ws` must be 256-byte aligned and at least the size returned
 *   by the matching *_workspace_size() function.  Its first
 *   SA_WS_HEADER_BYTES bytes are the header: the status block (the first
 *   256 bytes) and the slice counters of sa_sparse_decode_attn's path for
 *   few rows per KV head.  Zero the header once when the workspace is
 *   allocated: the library only ever writes a non-zero code into the status
 *   block (so the status is sticky until sa_clear_device_status(), which
 *   zeroes the whole header), and every launch leaves the counters it used
 *   at zero when it ends.  The rest is scratch owned by the call while it
 *   runs on `stream`: calls that overlap on the GPU must not share one
 *   workspace.
 * - Between calls the library keeps only per-device facts it looks up once
 *   (the driver's tensor-map entry point, the SM count, the largest cluster
 *   the top-k kernel can be scheduled with, which kernels have had their
 *   shared-memory limit raised), per host thread the last 16 tensor maps it
 *   encoded (each a function of an address and a shape only), and the fixed
 *   scratch array of
 *   sa_block_union_prefill_noalloc (see there); the workspace entry points
 *   are reentrant and thread-safe.
 */
#ifndef CROSS_LAYER_SHARED_SA_H
#define CROSS_LAYER_SHARED_SA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int sa_status;
#define SA_OK 0
#define SA_ERR_INVALID_ARG 1 /* bad pointer, size, shape or alignment          */
#define SA_ERR_UNSUPPORTED 2 /* valid request this build does not implement    */
#define SA_ERR_WORKSPACE 3   /* workspace missing, misaligned or too small      */
#define SA_ERR_CUDA 4        /* a CUDA runtime call failed (launch, attribute)  */
#define SA_ERR_TIMEOUT 5     /* device: a bounded wait gave up                  */
#define SA_ERR_DEVICE 6      /* device: an input value was out of range         */

typedef enum { SA_BF16 = 0, SA_F32 = 1 } sa_dtype;

#define SA_WS_HEADER_BYTES 4096

/* Human-readable name of a status code (static string). */
const char* sa_status_string(sa_status status);

/* Detail of the last failing call made by this thread ("" if none). */
const char* sa_last_error(void);

/* ABI version of this header: 1. */
int sa_abi_version(void);

/*
 * Synchronises `stream`, then copies the status block's first word into
 * *device_status (SA_OK, SA_ERR_TIMEOUT or SA_ERR_DEVICE) and, when
 * `detail` is not NULL, four detail words (kernel id, element index, value,
 * bound) into detail[0..3].  Returns SA_ERR_CUDA if the copy failed.
 */
sa_status sa_read_device_status(const void* ws, void* stream, int* device_status, int64_t* detail);

/* Enqueues a reset of the status block to zero on `stream`. */
sa_status sa_clear_device_status(void* ws, void* stream);

/* Self-test of the bounded waits every kernel of this library uses (not part
 * of the method; the pages have no counterpart).  Launches one CTA that
 * waits on an mbarrier nothing ever arrives on, through the same wait
 * routine the kernels use, with a limit of `limit_ns` nanoseconds instead of
 * the kernels' 1 s.  The wait gives up and records SA_ERR_TIMEOUT in the
 * status block of `ws` with detail (kernel id 8, 0, 0, limit_ns); no copy or
 * tensor-core operation is in flight when it does, and the kernel returns
 * normally, so the context stays usable.  1e3 <= limit_ns <= 1e9.
 * ws: at least SA_WS_HEADER_BYTES, 256-byte aligned. */
sa_status sa_wait_probe(void* ws, size_t ws_bytes, unsigned long long limit_ns, void* stream);

/* ------------------------------------------------------------------------
 * Indexer score, decode form  [IC section 1: the lightning indexer scores
 * every previous token for the current query; CLSA "Comment CLSA
 * fonctionne": the shared indexer layer computes the scores once].
 *
 * The pages name the DSA lightning indexer but print no formula; this call
 * computes its DSA form, one key vector per token shared by every indexer
 * head:
 *   scores[b*ld + t] = sum_j w[b,j] * max(0, sum_c qI[b,j,c] * KI[seq_off[b]+t, c])
 * for t in [0, seq_len[b]), with fp32 accumulation; the result is canonical
 * (+0, never -0).  Entries t >= seq_len[b] are left untouched.
 *
 *   qI       bf16 [B, H_I, d_I]       query of sequence b, one row per head
 *   w        fp32 [B, H_I]            head weights (positive in the method)
 *   KI       bf16 [n_tokens, d_I]     packed indexer-key cache
 *   seq_off  int64 [B+1] (device)     first KI row of sequence b
 *   seq_len  int32 [B]   (device)     visible keys of sequence b (<= S_max)
 *   S_max    host upper bound on seq_len (sizes the grid); ld >= S_max
 *   scores   fp32 [B, ld]
 * Supported: 1 <= H_I <= 64, d_I in {64, 128, 192, 256}.
 * Device errors: seq_len[b] > S_max or a row past n_tokens -> SA_ERR_DEVICE
 * (rows past n_tokens read as zero; nothing past column S_max is written).
 * ---------------------------------------------------------------------- */
size_t sa_index_score_workspace_size(int B);
sa_status sa_index_score(const void* qI, const float* w, const void* KI, const int64_t* seq_off,
                         const int32_t* seq_len, int B, int64_t n_tokens, int S_max, int H_I,
                         int d_I, float* scores, int64_t ld, void* ws, size_t ws_bytes,
                         void* stream);

/* ------------------------------------------------------------------------
 * Indexer score, chunked-prefill form  [same definition, IC section 1;
 * CA "Enonce du Probleme": queries of the current chunk attend to the
 * accumulated KV cache].  Nq queries of ONE sequence; query p sees keys
 * t in [0, q_pos[p]]:
 *   scores[p*ld + t] = sum_j w[p,j] * max(0, sum_c qI[p,j,c] * KI[t,c])
 *
 *   qI bf16 [Nq, H_I, d_I]; w fp32 [Nq, H_I]; KI bf16 [S, d_I];
 *   q_pos int32 [Nq] (device), each in [0, S); max_pos = host upper bound
 *   of q_pos (< S); scores fp32 [Nq, ld] with ld >= max_pos + 1.
 * Supported: 1 <= H_I <= 64, d_I in {64, 128, 192, 256} (as sa_index_score),
 * 0 <= Nq <= 4096 (Nq = 0 returns SA_OK without a launch).
 * Device errors: q_pos out of [0, max_pos] -> SA_ERR_DEVICE, row skipped.
 * ---------------------------------------------------------------------- */
size_t sa_index_score_prefill_workspace_size(int Nq);
sa_status sa_index_score_prefill(const void* qI, const float* w, const void* KI,
                                 const int32_t* q_pos, int Nq, int S, int max_pos, int H_I,
                                 int d_I, float* scores, int64_t ld, void* ws, size_t ws_bytes,
                                 void* stream);

/* The prefill indexer followed by the per-query top-k, with the same result
 * as sa_index_score_prefill then sa_topk (n_valid = q_pos + 1, n_max =
 * max_pos + 1), writing no scores for the caller: the queries run in blocks
 * of rows_per_block (0: all Nq in one block), each block's scores written to
 * the workspace and selected before the next block is scored.  The
 * workspace then holds rows_per_block x S fp32 scores.  Every block streams
 * all key tiles again, so smaller blocks trade time for workspace (c4,
 * S = 131072, 2048 queries: 1.93 ms in one block, 3.0 ms in blocks of 1024,
 * 5.4 ms of 512, 18.9 ms of 128).
 *   idx  int32 [Nq, k] out, as sa_topk writes it (ascending, -1 padded)
 * Other arguments and device errors as sa_index_score_prefill and sa_topk.
 * Workspace: sa_index_topk_prefill_workspace_size (the same rows_per_block). */
size_t sa_index_topk_prefill_workspace_size(int Nq, int S, int max_pos, int k, int rows_per_block);
sa_status sa_index_topk_prefill(const void* qI, const float* w, const void* KI, const int32_t* q_pos,
                                int Nq, int S, int max_pos, int H_I, int d_I, int k,
                                int rows_per_block, int32_t* idx, void* ws, size_t ws_bytes,
                                void* stream);

/* ------------------------------------------------------------------------
 * Top-k  [IC section 1: keep the k most relevant tokens; CLSA: the top-k
 * selection runs once and its index is reused].
 *
 * Row q of `scores` has n_valid[q] valid entries.  Selects the min(k,
 * n_valid[q]) largest; ties go to the LOWER index; the order on floats is
 * IEEE with -0 == +0 (NaN inputs give an unspecified, in-range result).
 *   idx        int32 [Nq, k]  selected indices in ASCENDING order, then -1
 *   top_scores fp32 [Nq, k]   (nullable) the matching scores, 0 for padding
 *   n_max      host upper bound of n_valid (<= ld)
 * Device errors: n_valid[q] outside [0, n_max] -> SA_ERR_DEVICE, clamped.
 * ---------------------------------------------------------------------- */
size_t sa_topk_workspace_size(int Nq, int n_max, int k);
sa_status sa_topk(const float* scores, int64_t ld, const int32_t* n_valid, int Nq, int n_max,
                  int k, int32_t* idx, float* top_scores, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Dynamic k by routing mass  [CLSA news article, sections "Le cout : limites
 * de compatibilite" and "Ce que cela signifie pour l'inference sur longs
 * contextes": the indexer layer could choose k per query instead of a fixed
 * k; the pages leave the rule open.  The reading here: a coverage target on
 * the routing scores' mass.]
 *
 * Row q (n = n_valid[q] scores) keeps the smallest number m of its tokens,
 * taken in sa_topk's order (score descending, ties to the lower index),
 * whose summed score reaches tau times the row's total score (the sum over
 * all n tokens), but at most k_max; a row whose top k_max never reaches it
 * keeps min(n, k_max).  Sums are fp64.  Meant for non-negative scores (the
 * routing weights of sa_indexer_layer_attn, or sa_index_score with positive
 * head weights): the running sum is then non-decreasing.
 *
 *   idx     int32 [Nq, k_max]   the m kept indices ascending, then -1
 *   counts  int32 [Nq]          m per row
 *   tau     in (0, 1]; 1 <= k_max <= 4096
 * Other arguments as sa_topk.  Runs sa_topk's kernels for the top k_max
 * (with their scores, into the workspace), then one CTA per row.
 * ---------------------------------------------------------------------- */
size_t sa_topk_dynamic_workspace_size(int Nq, int n_max, int k_max);
sa_status sa_topk_dynamic(const float* scores, int64_t ld, const int32_t* n_valid, int Nq, int n_max,
                          int k_max, double tau, int32_t* idx, int32_t* counts, void* ws, size_t ws_bytes,
                          void* stream);

/* ------------------------------------------------------------------------
 * Sparse decode attention for one layer group  [IC section 1: main
 * attention over the k selected tokens; IC section 2: S layers reuse the
 * top-k index of the nearest upstream F layer; CLSA "Comment CLSA
 * fonctionne": the same index is handed to every cross-decoder layer over
 * the shared KV cache].
 *
 * For layer l < L_g, sequence b, query head h (KV head g = h / (Hq/Hkv)):
 *   z_t = scale * Q[l,b,h,:] . K_b[g,t,:],  t in idx[b,:] (entries < 0 skipped)
 *   O[l,b,h,:] = sum_t softmax(z)_t * V_b[g,t,:]      (fp32 softmax/accumulate)
 * A row with no valid index gets O = 0.
 *
 *   Q        bf16 [L_g, B, Hq, d]   queries of every layer of the group
 *   K, V     bf16 packed per sequence: sequence b starts at element
 *            seq_off[b]*Hkv*d and is laid out [Hkv, seq_len[b], d]
 *            (KV-head-major); every layer of the group reads this cache
 *   seq_off  int64 [B+1], seq_len int32 [B] (device)
 *   n_tokens rows of the packed cache per KV head (sum of seq_len); the
 *            caches hold n_tokens * Hkv rows of d elements
 *   idx      int32 [B, k] (device) shared index of the group
 *   O        [L_g, B, Hq, d], bf16 or fp32 per out_dtype
 * Each selected K/V row is brought from HBM once per (sequence, KV head)
 * for the whole group.  Supported: d = 128, Hq % Hkv == 0, Hq/Hkv <= 128.
 * Two kernels: with L_g * Hq/Hkv > 8 rows per (sequence, KV head), 128-row
 * tensor-core tiles (tcgen05; P rounded to bf16 for bf16 outputs, split in
 * two bf16 parts for fp32 outputs); with at most 8 (one layer of a
 * per-layer decoder), warp-level 16-row MMA tiles with P always split in
 * two bf16 parts.  The second kernel splits the index entries of a
 * (sequence, KV head) over several CTAs whose partials meet in the
 * workspace scratch, counted on counters in the workspace header.
 * Device errors: idx entry >= seq_len[b] -> SA_ERR_DEVICE, entry skipped;
 * a bounded wait that gave up -> SA_ERR_TIMEOUT.
 * ---------------------------------------------------------------------- */
size_t sa_sparse_decode_attn_workspace_size(int L_g, int B, int Hq, int Hkv, int d, int k);
sa_status sa_sparse_decode_attn(const void* Q, const void* K, const void* V, const int64_t* seq_off,
                                const int32_t* seq_len, const int32_t* idx, int L_g, int B,
                                int64_t n_tokens, int Hq, int Hkv, int d, int k, float scale, void* O,
                                sa_dtype out_dtype, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * The CLSA indexer layer read as a full attention layer whose attention
 * weights route the shared index  [CLSA news article, section "La
 * precision reste stable": the routing index is computed once from the
 * attention scores of the indexer layer, which sees the same query state
 * and cache as every other layer].  The pages give no formula for the
 * aggregation over heads; this reads it as the sum of the attention weights.
 *
 * For sequence b, query head h (KV head g = h / (Hq/Hkv)), every cached
 * token t < seq_len[b]:
 *   z[h,t] = scale * Q[b,h,:] . K_b[g,t,:],   p[h,t] = softmax_t z[h,t]
 *   O[b,h,:]     = sum_t p[h,t] * V_b[g,t,:]        (the layer's dense output)
 *   scores[b,t]  = sum_h p[h,t]                     (fp32 routing score)
 * sa_topk(scores, seq_len, ...) then gives the index the later layers share.
 *
 *   Q        bf16 [B, Hq, d]: the indexer layer's queries
 *   K, V     packed cache as in sa_sparse_decode_attn
 *   seq_off  int64 [B+1], seq_len int32 [B] (device); S_max >= every seq_len
 *   O        [B, Hq, d], bf16 or fp32 per out_dtype
 *   scores   fp32 [B, ld], ld >= S_max; entries t >= seq_len[b] untouched
 * Supported: d = 128, Hq/Hkv in {1, 2, 4, 8}, Hq <= 256.  The workspace
 * holds the logits (B*Hq*S_max fp32) and per-2048-key partial results.
 * Device errors: seq_len[b] outside [0, S_max] or past n_tokens ->
 * SA_ERR_DEVICE, the sequence is treated as empty.
 * ---------------------------------------------------------------------- */
size_t sa_indexer_layer_attn_workspace_size(int B, int S_max, int Hq, int Hkv, int d);
sa_status sa_indexer_layer_attn(const void* Q, const void* K, const void* V, const int64_t* seq_off,
                                const int32_t* seq_len, int B, int64_t n_tokens, int S_max, int Hq,
                                int Hkv, int d, float scale, void* O, sa_dtype out_dtype,
                                float* scores, int64_t ld, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * One decode step over a layer pattern  [IC section 2: a binary pattern
 * marks F layers, which run their indexer and overwrite the cached top-k
 * index, and S layers, which reuse the index of the nearest upstream F
 * layer - one conditional branch in the inference loop, no extra memory].
 *
 * pattern: n_layers characters 'F' / 'S', first one 'F'.  Host arrays of
 * device pointers, one entry per layer: qI[l], w[l], KI[l] (read for F
 * layers only, shapes as in sa_index_score) and K[l], V[l] (the cache that
 * layer reads, layout as in sa_sparse_decode_attn).  Q / O: [n_layers, B,
 * Hq, d].  idx [B, k] is the index cache (overwritten at every F layer) and
 * scores [B, ld] the indexer's scratch output.  Consecutive layers that
 * share one index and one cache run as a single fused group call.
 * ---------------------------------------------------------------------- */
size_t sa_decode_step_workspace_size(int n_layers, int B, int S_max, int Hq, int Hkv, int d, int k);
sa_status sa_decode_step(const char* pattern, int n_layers, const void* const* qI,
                         const float* const* w, const void* const* KI, const void* const* K,
                         const void* const* V, const int64_t* seq_off, const int32_t* seq_len,
                         int B, int64_t n_tokens, int S_max, int H_I, int d_I, int k, const void* Q,
                         int Hq, int Hkv, int d, float scale, void* O, sa_dtype out_dtype,
                         int32_t* idx, float* scores, int64_t ld, void* ws, size_t ws_bytes,
                         void* stream);

/* ------------------------------------------------------------------------
 * The decode step with the new token appended to the caches, and/or one
 * attention launch per layer.  The pages define neither; they are the steps
 * either side of the shared-index path in a real decoder: the new token's
 * indexer key and K/V rows enter the caches before they are searched, and
 * layer l+1's queries only exist after layer l has run.
 *
 * Same arguments as sa_decode_step, plus:
 *   new_KI  host array (n_layers entries, read at F layers; or NULL: no
 *           append): device pointer to [B, d_I] bf16, the new token's
 *           indexer key of every sequence.  It is written to row
 *           seq_off[b] + seq_len[b] - 1 of KI[l] (seq_len counts the new
 *           token) and its score is computed from this fresh row.
 *   new_K, new_V  host arrays (or both NULL): device pointers to [B, Hkv, d]
 *           bf16, the new token's K / V rows, written to position
 *           seq_len[b] - 1 of every head of the cache K[l], V[l] of each F
 *           layer.  Every S layer must then read its F layer's cache
 *           (SA_ERR_UNSUPPORTED otherwise).  Needs new_KI.
 *   flags   0, or SA_STEP_PER_LAYER: one attention launch per layer, no
 *           fusion of a group's layers (each layer's queries are ready only
 *           after the previous layer in a real model).  Results are the same
 *           either way.
 * KI, K and V are written, hence non-const.  All new rows 16-byte aligned.
 * ---------------------------------------------------------------------- */
#define SA_STEP_PER_LAYER 1
sa_status sa_decode_step_ex(const char* pattern, int n_layers, const void* const* qI,
                            const float* const* w, void* const* KI, void* const* K, void* const* V,
                            const void* const* new_KI, const void* const* new_K,
                            const void* const* new_V, const int64_t* seq_off,
                            const int32_t* seq_len, int B, int64_t n_tokens, int S_max, int H_I,
                            int d_I, int k, const void* Q, int Hq, int Hkv, int d, float scale,
                            void* O, sa_dtype out_dtype, int32_t* idx, float* scores, int64_t ld,
                            int flags, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Block union + zero-copy paged causal attention for one prefill chunk
 * [CA selection step: map each selected token to its KV block, union over
 * the query blocks of the chunk (Q-block union) and over the query heads
 * of each GQA group (intra-group union) into a minimal per-group table
 * T_g that keeps every selected block; CA execution step: the table goes
 * to a dense paged attention kernel as kv_indptr / kv_indices and the
 * blocks are read in place from the KV-head-major cache, no copy].
 *
 *   idx        int32 [Nq, k]  per-query selected tokens (entries < 0 skipped)
 *   q_pos      int32 [Nq]     position of each query (causal limit)
 *   Q          bf16 [Nq, Hq, d];  K, V bf16 [Hkv, S, d]
 *   kv_indptr  int32 [Hkv + 1]           (output) CSR row pointers
 *   kv_indices int32 [Hkv * ceil(S/block)] (output) sorted distinct blocks
 *   O          [Nq, Hq, d] bf16 / fp32: query p, head h attends with
 *              softmax to every key t in the blocks of T_{h/(Hq/Hkv)} with
 *              t <= q_pos[p] and t < S.
 * The selection is shared by all heads, so every group's table is the
 * same set.  Supported: d = 128, block = 64.
 * ---------------------------------------------------------------------- */
size_t sa_block_union_prefill_workspace_size(int S, int Nq, int Hq, int Hkv, int d, int k, int block);
sa_status sa_block_union_prefill(const int32_t* idx, const int32_t* q_pos, const void* Q,
                                 const void* K, const void* V, int S, int Nq, int Hq, int Hkv,
                                 int d, int k, int block, float scale, int32_t* kv_indptr,
                                 int32_t* kv_indices, void* O, sa_dtype out_dtype, void* ws,
                                 size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * sa_block_union_prefill without a workspace.  The pages have no
 * counterpart: this entry point exists for callers that cannot allocate
 * device memory around the call - code running inside a CUDA graph capture
 * (where cudaMalloc is not allowed), runtimes without a device allocator
 * hook, or a host that has handed all memory to another pool.
 *
 * Same arguments, results and device-side skipping as
 * sa_block_union_prefill, minus ws / ws_bytes.  Its scratch (a status block
 * and one byte per KV block) is a fixed array inside libsa's own device
 * memory, SA_NOALLOC_MAX_KV_BLOCKS bytes plus 256, held by every GPU that
 * loads the library until the process exits.  Limits:
 *   - ceil(S / block) <= SA_NOALLOC_MAX_KV_BLOCKS (S <= 2,097,152 at block 64),
 *     larger S returns SA_ERR_UNSUPPORTED before anything is enqueued;
 *   - the first call on each device looks up the array's device address, so
 *     make that first call before any stream capture begins;
 *   - that address is kept for the life of the process: do not call this
 *     entry point on a device after a reset of it (cudaDeviceReset or a
 *     primary-context reset), which would leave the kept address stale;
 *   - every call shares the one array: calls that may overlap on the GPU
 *     (different streams, or different host threads on one device) race and
 *     must be ordered by the caller;
 *   - device-side range errors are skipped as usual, but their record stays
 *     in the library's array (cleared at every call) and is not reported.
 * Allocates nothing: no cudaMalloc / cudaFree, no allocating library call.
 * ---------------------------------------------------------------------- */
#define SA_NOALLOC_MAX_KV_BLOCKS 32768
sa_status sa_block_union_prefill_noalloc(const int32_t* idx, const int32_t* q_pos, const void* Q,
                                         const void* K, const void* V, int S, int Nq, int Hq, int Hkv,
                                         int d, int k, int block, float scale, int32_t* kv_indptr,
                                         int32_t* kv_indices, void* O, sa_dtype out_dtype, void* stream);

/* ------------------------------------------------------------------------
 * Priority-ordered block execution with early skipping for a prefill chunk
 * [CoSA lay summary: a kernel-aware proxy hands the attention kernel a
 * priority list of blocks instead of a yes/no list; the ordered-skipping
 * kernel reads the blocks in that order, builds a progressive score from
 * the most important ones first and then skips the rest].  The pages give
 * neither the proxy's formula nor the skip rule; the readings built here:
 *
 * sa_kap_order (the proxy): for query block i (queries i*q_block ..
 * i*q_block + q_block - 1; the last block may be shorter), block B's hit
 * count is the number of entries idx[p, e] of those queries with
 * 0 <= idx[p,e] < S and idx[p,e] / block == B.  order[i, 0 : nT] is the
 * union table kv_indices[kv_indptr[0] : kv_indptr[1]] (nT blocks, the
 * table of group 0; every group's table is the same set) ordered by hit
 * count, larger first, equal counts by ascending block id.
 *   idx        int32 [Nq, k]
 *   order      int32 [ceil(Nq / q_block), ld], ld >= ceil(S / block);
 *              entries past nT of each row are not written
 * Supported: ceil(S / block) <= 16384.  A table entry outside
 * [0, ceil(S/block)) is reported (SA_ERR_DEVICE, kernel id 5) and ranked
 * with count 0; a table longer than ceil(S/block) entries is reported the
 * same way (entry -1) and only its first ceil(S/block) entries are ordered.  Workspace: sa_kap_order_workspace_size() bytes (the
 * status block).
 *
 * sa_osk_prefill (union, proxy and ordered-skipping attention in one
 * call): the block union of sa_block_union_prefill (kv_indptr,
 * kv_indices), then sa_kap_order with q_block = 128 / (Hq / Hkv) (one
 * query block fills the 128 rows of an attention tile), then attention
 * per unit (query block i, KV group g) - the rows (p, h) of the block's
 * queries and the group's heads:
 *   step n = blocks order[i][2n] and order[i][2n+1] (128 keys);
 *   after step n, a row's share is the weight its visible keys in the
 *   step add to its softmax, relative to its running sum over steps
 *   0..n (+inf while it has seen no key); the first step where every row
 *   of the unit has a share below tau ends the unit two steps later (the
 *   steps already in flight finish); N = min(steps in the list, that
 *   step + 3), or all steps when no step qualifies;
 *   O[p, h] = softmax attention of row (p, h) over its visible keys
 *   (t <= q_pos[p], t < S) of steps 0..N-1.
 * tau = 0 never skips: O equals sa_block_union_prefill's output.
 *   order      int32 [ceil(Nq*G/128), ceil(S/block)] (output, G = Hq/Hkv)
 *   steps      int32 [Hkv * ceil(Nq*G/128)] (output): N of unit
 *              g * ceil(Nq*G/128) + i
 * Other arguments and outputs as in sa_block_union_prefill.  Supported:
 * d = 128, block = 64, G dividing 128, ceil(S/block) <= 16384.
 * Workspace: sa_osk_prefill_workspace_size bytes.
 * ---------------------------------------------------------------------- */
size_t sa_kap_order_workspace_size(void);
sa_status sa_kap_order(const int32_t* idx, int Nq, int k, int S, int block, int q_block,
                       const int32_t* kv_indptr, const int32_t* kv_indices, int32_t* order,
                       int64_t ld, void* ws, size_t ws_bytes, void* stream);
size_t sa_osk_prefill_workspace_size(int S, int Nq, int Hq, int Hkv, int d, int k, int block);
sa_status sa_osk_prefill(const int32_t* idx, const int32_t* q_pos, const void* Q, const void* K,
                         const void* V, int S, int Nq, int Hq, int Hkv, int d, int k, int block,
                         float scale, float tau, int32_t* kv_indptr, int32_t* kv_indices,
                         int32_t* order, int32_t* steps, void* O, sa_dtype out_dtype, void* ws,
                         size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Context-parallel decode: one sequence's context sharded over N ranks
 * [CLSA news article, section "Ce que cela signifie pour l'inference sur
 * longs contextes": how the method behaves past 128K tokens is left open.
 * The pages have no sharding scheme.  This one is the plainest that gives
 * the same result as one GPU.]
 *
 * Rank r holds a contiguous slice of every sequence (tokens [lo_r, hi_r),
 * slices in rank order, possibly empty) as its own packed caches.  A step:
 *   1. sa_index_score + sa_topk (with top_scores) over the local slice;
 *   2. all ranks' (top_scores, idx) gathered, rank-major, on every rank;
 *   3. sa_cp_select: the global top-k of those candidates, mapped back to
 *      this rank's local indices;
 *   4. sa_sparse_decode_attn_partial over the local selected rows;
 *   5. all ranks' (O_part, ml) gathered; sa_combine_partials.
 * A token of the global top-k is in its slice's top-k.  Candidate position
 * order (rank-major, then ascending local index) is ascending global
 * index, so the tie rule (lower index first) carries over.  Softmax over a
 * union of disjoint key sets is the log-sum-exp merge of the parts.  The
 * step therefore selects the same index as sa_decode_step on one GPU, and
 * attends over it.
 * ---------------------------------------------------------------------- */

/* The sparse decode attention of one rank, left unnormalised.  Arguments as
 * sa_sparse_decode_attn, plus idx_count (nullable, device int32 [B]): when
 * set, only the first idx_count[b] entries of idx row b (clamped to [0, k])
 * are read, the rest counting as padding, and the keys are split over that
 * many, so a rank whose
 * share of the index is small runs on only that share.  For each row
 * (l, b, h), with a reference m (log2
 * units) at most 8 below max_t z_t * log2(e) over its valid selected keys:
 *   O_part[row, :] = sum_t 2^(z_t*log2(e) - m) V_t    fp32 [L_g, B, Hq, d]
 *   ml[row]        = (m, sum_t 2^(z_t*log2(e) - m))   fp32 pairs [L_g, B, Hq]
 * so O_part / l is the row's output and m + log2(l) its log-sum-exp in log2
 * units; m itself is whatever reference the kernel kept.  A row with no
 * valid index gets l = 0 and O_part = 0.  ml must be 8-byte aligned.
 * Workspace: sa_sparse_decode_attn_workspace_size. */
sa_status sa_sparse_decode_attn_partial(const void* Q, const void* K, const void* V,
                                        const int64_t* seq_off, const int32_t* seq_len,
                                        const int32_t* idx, int L_g, int B, int64_t n_tokens, int Hq,
                                        int Hkv, int d, int k, const int32_t* idx_count, float scale,
                                        float* O_part, float* ml, void* ws, size_t ws_bytes,
                                        void* stream);

/* The global top-k by exchanging histograms (the context-parallel step's
 * selection; replaces steps 1-3 above after the local sa_index_score).
 * Scores map to 32-bit keys ordered like the floats (-0 == +0); the k-th
 * largest key T over all ranks is found digit by digit, key bits [31:20],
 * [19:8], [7:0], each digit the one where the count of larger keys summed
 * over the ranks' histograms first reaches the number still needed (the
 * radix select of sa_topk, with the ranks' histograms summed).  A rank then
 * keeps its keys above T and, of its keys equal to T, those the lower-index
 * rule gives it: slices are in rank order, so ties go to the lower ranks,
 * then to the lower local indices.  The union over ranks is exactly
 * sa_topk's selection over the whole context (all valid keys when there
 * are at most k).  A step, every rank alike:
 *   sa_cp_radix_level(level 0) -> hist [B][4096]; all-gather (rank-major);
 *   sa_cp_radix_level(level 1, the gathered level-0 histograms) -> [B][4096];
 *   all-gather; sa_cp_radix_level(level 2, gathered level 1) -> [B][256];
 *   all-gather; sa_cp_radix_select(the gathered level-2 histograms).
 *   scores     fp32 [B, ld]: this rank's indexer scores over its slice,
 *              entries [0, n_local[b]) of row b
 *   n_local    int32 [B] (device): this rank's slice length per sequence
 *   gathered   every rank's histograms of the previous level, rank r's
 *              [B][bins] block at element offset r * rank_stride (bins 4096
 *              for levels 0 and 1, 256 for level 2); NULL at level 0
 *   hist_out   int32 [B][4096] (levels 0, 1) or [B][256] (level 2)
 *   local_idx  int32 [B, k] out: this rank's entries of the global top-k,
 *              as local indices, ascending, then -1
 *   local_count int32 [B] out (nullable): their number (the idx_count of
 *              sa_sparse_decode_attn_partial)
 * The workspace (sa_cp_radix_workspace_size, one per rank) carries the
 * per-sequence state from each call to the next: keep it for the step's
 * four calls.  1 <= N <= 1024.  Device errors: n_local[b] < 0 ->
 * SA_ERR_DEVICE, the row counts as empty.  One CTA of 1024 threads per
 * sequence per call. */
size_t sa_cp_radix_workspace_size(int B);
sa_status sa_cp_radix_level(const float* scores, int64_t ld, const int32_t* n_local, int B, int k, int N,
                            int level, const int32_t* gathered, int64_t rank_stride, int32_t* hist_out,
                            void* ws, size_t ws_bytes, void* stream);
sa_status sa_cp_radix_select(const float* scores, int64_t ld, const int32_t* n_local, int B, int k, int N,
                             int rank, const int32_t* gathered, int64_t rank_stride, int32_t* local_idx,
                             int32_t* local_count, void* ws, size_t ws_bytes, void* stream);

/* Global top-k over the gathered candidates.
 *   cand_scores, cand_idx  rank r's top_scores (fp32 [B, k]) and idx (int32
 *               [B, k]) from sa_topk over its slice: each idx row ascending,
 *               then -1 padding, as sa_topk writes it (other orders give
 *               unspecified, in-bounds results), at
 *               element offset r * cand_stride of each (so one all-gathered
 *               buffer of [N][scores | idx] blocks serves both, with
 *               cand_idx = cand_scores + B*k and cand_stride = 2*B*k)
 *   local_idx   int32 [B, k] out: the global top-k entries in rank `rank`'s
 *               slice, as its local indices, ascending, then -1
 *   local_count int32 [B] out (nullable): the number of those entries, the
 *               idx_count of sa_sparse_decode_attn_partial
 * The selection is sa_topk's (min(k, candidates) largest, ties to the lower
 * position) over the N*k candidates of each sequence, padding scoring -inf.
 * 0 <= rank < N; N*k <= 2^31 - 1; cand_stride >= B*k when N > 1. */
size_t sa_cp_select_workspace_size(int N, int B, int k);
sa_status sa_cp_select(const float* cand_scores, const int32_t* cand_idx, int64_t cand_stride, int N,
                       int B, int k, int rank, int32_t* local_idx, int32_t* local_count, void* ws,
                       size_t ws_bytes, void* stream);

/* The log-sum-exp merge of P partial results of the same rows:
 *   O[row, :] = sum_p 2^(m_p - M) O_part_p[row, :] / sum_p 2^(m_p - M) l_p,
 * with M the largest m_p among parts with l_p > 0; O = 0 where every l_p = 0.
 *   O_part_p  fp32 [rows, d] at O_part + p * o_stride (floats)
 *   (m_p, l_p) fp32 pairs [rows] at ml + p * ml_stride (floats)
 *   O         [rows, d] in out_dtype (bf16 or fp32)
 * With P > 1: o_stride >= rows*d and a multiple of 4, ml_stride >= 2*rows
 * and even (one all-gathered buffer of [P][O_part | ml] blocks: ml = O_part
 * + rows*d, both strides rows*(d+2) rounded up to a multiple of 4).
 * Supported: d = 128, 1 <= P.  rows = 0
 * returns SA_OK without a launch.  No workspace. */
sa_status sa_combine_partials(const float* O_part, int64_t o_stride, const float* ml, int64_t ml_stride,
                              int P, int64_t rows, int d, void* O, sa_dtype out_dtype, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* CROSS_LAYER_SHARED_SA_H */
