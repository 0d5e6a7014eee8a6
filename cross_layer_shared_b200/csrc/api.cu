// C ABI of libsa (declared in include/sa.h): host-side argument checks,
// tensor-map encoding, workspace carving and kernel launches.  Every check
// runs before anything is enqueued; nothing here allocates device memory.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdarg.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <cmath>
#include <mutex>
#include <string>

#include "../../include/sa.h"
#include "attn.cuh"
#include "sm100.cuh"
#include "indexer.cuh"
#include "route_attn.cuh"
#include "cp.cuh"
#include "status.cuh"
#include "topk.cuh"
#include "union.cuh"

namespace sa {

namespace {
std::mutex g_attr_mu;
struct AttrEntry {
  int dev;
  const void* fn;
};
AttrEntry g_attr[256];
int g_attr_n = 0;
}  // namespace

bool smem_attr_done(int dev, const void* fn) {
  std::lock_guard<std::mutex> lk(g_attr_mu);
  for (int i = 0; i < g_attr_n; ++i)
    if (g_attr[i].dev == dev && g_attr[i].fn == fn) return true;
  return false;
}

void smem_attr_mark(int dev, const void* fn) {
  std::lock_guard<std::mutex> lk(g_attr_mu);
  if (g_attr_n < 256) g_attr[g_attr_n++] = {dev, fn};
}

}  // namespace sa

namespace {

thread_local std::string g_last_error;

sa_status fail(sa_status code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

sa_status cuda_fail(const char* where, cudaError_t e) {
  return fail(SA_ERR_CUDA, "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int num_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  static std::atomic<int> cache[64];  // per device; every writer stores the same value
  if (dev >= 0 && dev < 64) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  if (dev >= 0 && dev < 64) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// A tensor map is a pure function of the address and the geometry, so the
// last few encoded per host thread are kept and reused (a decode step encodes
// the same five every call).
struct TmapKey {
  const void* base;
  int rank;
  uint64_t dims[3], strides[2];
  uint32_t box[3];
  bool operator==(const TmapKey& o) const { return memcmp(this, &o, sizeof *this) == 0; }
};
struct TmapEntry {
  TmapKey key;
  CUtensorMap map;
  bool used;
};
constexpr int kTmapCache = 16;
thread_local TmapEntry g_tmap_cache[kTmapCache];
thread_local int g_tmap_next = 0;

// bf16 tensor map with 128-byte swizzle; dims innermost first (elements),
// strides in bytes for dims 1.. ; box in elements.
sa_status make_tmap(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const uint64_t* strides,
                    const uint32_t* box) {
  TmapKey key;
  memset(&key, 0, sizeof key);  // padding included: the key compares as bytes
  key.base = base;
  key.rank = rank;
  for (int i = 0; i < rank && i < 3; ++i) {
    key.dims[i] = dims[i];
    key.box[i] = box[i];
    if (i + 1 < rank) key.strides[i] = strides[i];
  }
  for (int i = 0; i < kTmapCache; ++i)
    if (g_tmap_cache[i].used && g_tmap_cache[i].key == key) {
      *m = g_tmap_cache[i].map;
      return SA_OK;
    }
  auto fn = encode_fn();
  if (!fn) return fail(SA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  uint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SA_ERR_INVALID_ARG, "tensor map encoding failed (CUresult %d)", (int)r);
  TmapEntry& e = g_tmap_cache[g_tmap_next];
  g_tmap_next = (g_tmap_next + 1) % kTmapCache;
  e.key = key;
  e.map = *m;
  e.used = true;
  return SA_OK;
}

// [rows, 128] bf16 as a 2-D tensor map with a 64 x 1 box (rows gathered four at a time)
sa_status make_rows_tmap(CUtensorMap* m, const void* base, int64_t rows) {
  if (rows < 1 || rows >= (1ll << 31)) return fail(SA_ERR_INVALID_ARG, "tensor of %lld rows: need 1 <= rows < 2^31", (long long)rows);
  const uint64_t dims[2] = {128, (uint64_t)rows};
  const uint64_t str[1] = {256};
  const uint32_t box[2] = {64, 1};
  return make_tmap(m, base, 2, dims, str, box);
}

// [rows, 128] bf16 as a 2-D tensor map with a 64 x 128 box (half the columns
// of a 128-row tile per load)
sa_status make_tile128_tmap(CUtensorMap* m, const void* base, int64_t rows) {
  if (rows < 1 || rows >= (1ll << 31)) return fail(SA_ERR_INVALID_ARG, "tensor of %lld rows: need 1 <= rows < 2^31", (long long)rows);
  const uint64_t dims[2] = {128, (uint64_t)rows};
  const uint64_t str[1] = {256};
  const uint32_t box[2] = {64, 128};
  return make_tmap(m, base, 2, dims, str, box);
}

// [rows, 128] bf16 as a 2-D tensor map with a 64 x 64 box (one 64-token KV
// block, half of its columns, per load)
sa_status make_block_tmap(CUtensorMap* m, const void* base, int64_t rows) {
  if (rows < 1 || rows >= (1ll << 31)) return fail(SA_ERR_INVALID_ARG, "tensor of %lld rows: need 1 <= rows < 2^31", (long long)rows);
  const uint64_t dims[2] = {128, (uint64_t)rows};
  const uint64_t str[1] = {256};
  const uint32_t box[2] = {64, 64};
  return make_tmap(m, base, 2, dims, str, box);
}

sa::DeviceStatus* status_of(void* ws) { return reinterpret_cast<sa::DeviceStatus*>(ws); }

sa_status check_ws(void* ws, size_t ws_bytes, size_t need, const char* who) {
  if (ws == nullptr) return fail(SA_ERR_WORKSPACE, "%s: workspace is NULL", who);
  if (!aligned(ws, 256)) return fail(SA_ERR_WORKSPACE, "%s: workspace must be 256-byte aligned", who);
  if (ws_bytes < need)
    return fail(SA_ERR_WORKSPACE, "%s: workspace of %zu bytes is below the %zu required", who, ws_bytes, need);
  return SA_OK;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int index_npad(int H_I) { return (H_I + 15) / 16 * 16; }

// ---- sparse attention split choice -----------------------------------------
struct AttnPlan {
  int n_mtiles, n_split, keys_per_split, units;
};

AttnPlan plan_decode_attn(int L_g, int B, int Hq, int Hkv, int k) {
  AttnPlan p;
  const int R = L_g * (Hq / Hkv);
  p.n_mtiles = (R + 127) / 128;
  const int base = B * Hkv * p.n_mtiles;
  const int max_split = (k + 127) / 128;
  int s = num_sms() / (base > 0 ? base : 1);
  if (s > max_split) s = max_split;
  if (s > 8) s = 8;
  int p2 = 1;  // splits form a cluster: 1, 2, 4 or 8 CTAs
  while (p2 * 2 <= s) p2 *= 2;
  s = p2;
  p.keys_per_split = (int)round_up((size_t)((k + s - 1) / s), 128);
  if (p.keys_per_split < 128) p.keys_per_split = 128;
  p.n_split = s;  // trailing splits may get no keys; they merge as empty
  p.units = base * p.n_split;
  return p;
}

// Key splits per prefill row tile (a cluster of 1, 2 or 4 CTAs, merged at the
// end): the fewest whose launch fills its last wave of one-CTA-per-SM units to
// within 5 %.  Every unit of a prefill chunk has about the same work (the
// union of blocks is shared), so a part-empty last wave idles SMs for a
// whole unit's time: c4's 512 units on 148 SMs are 3.46 waves (86 % busy),
// split in two 6.92 waves (99 %).
int prefill_split(int units) {
  const int sms = num_sms();
  int best = 1;
  double best_eff = 0.0;
  for (int s = 1; s <= 4; s *= 2) {
    const double waves = (double)units * s / sms;
    const double eff = waves / std::ceil(waves);
    if (eff > best_eff + 0.05) {
      best = s;
      best_eff = eff;
    }
  }
  return best;
}

size_t attn_ws_bytes(const AttnPlan& p) {
  (void)p;
  return SA_WS_HEADER_BYTES;
}

sa_status validate_index(const void* qI, const float* w, const void* KI, int H_I, int d_I, const char* who) {
  if (!qI || !w || !KI) return fail(SA_ERR_INVALID_ARG, "%s: NULL tensor pointer", who);
  if (H_I < 1 || H_I > 64) return fail(SA_ERR_UNSUPPORTED, "%s: H_I=%d outside [1, 64]", who, H_I);
  if (d_I != 64 && d_I != 128 && d_I != 192 && d_I != 256)
    return fail(SA_ERR_UNSUPPORTED, "%s: d_I=%d not in {64, 128, 192, 256}", who, d_I);
  if (!aligned(qI, 16) || !aligned(KI, 16)) return fail(SA_ERR_INVALID_ARG, "%s: qI and KI must be 16-byte aligned", who);
  if (!aligned(w, 4)) return fail(SA_ERR_INVALID_ARG, "%s: w must be 4-byte aligned", who);
  return SA_OK;
}

sa_status run_index_decode(const void* qI, const float* w, const void* KI, const int64_t* seq_off,
                           const int32_t* seq_len, int B, int64_t n_tokens, int S_max, int H_I, int d_I,
                           float* scores, int64_t ld, void* ws, cudaStream_t stream,
                           const sa::AppendArgs& ap = sa::AppendArgs{}) {
  CUtensorMap tm_ki, tm_qi;
  {
    const uint64_t dims[2] = {(uint64_t)d_I, (uint64_t)n_tokens};
    const uint64_t str[1] = {(uint64_t)d_I * 2};
    const uint32_t box[2] = {64, 128};
    sa_status st = make_tmap(&tm_ki, KI, 2, dims, str, box);
    if (st != SA_OK) return st;
  }
  const int npad = index_npad(H_I);
  {
    const uint64_t dims[3] = {(uint64_t)d_I, (uint64_t)H_I, (uint64_t)B};
    const uint64_t str[2] = {(uint64_t)d_I * 2, (uint64_t)H_I * d_I * 2};
    const uint32_t box[3] = {64, (uint32_t)npad, 1};
    sa_status st = make_tmap(&tm_qi, qI, 3, dims, str, box);
    if (st != SA_OK) return st;
  }
  sa::IndexerArgs a{w, seq_off, seq_len, B, n_tokens, S_max, H_I, d_I, scores, ld, status_of(ws), ap};
  cudaError_t e = sa::launch_indexer_decode(a, tm_ki, tm_qi, npad, num_sms(), stream);
  if (e != cudaSuccess) return cuda_fail("sa_index_score launch", e);
  return SA_OK;
}

__global__ void prefill_rows_kernel(const int32_t* __restrict__ q_pos, int Nq, int max_pos, int64_t* seq_off,
                                    int32_t* seq_len, sa::DeviceStatus* status) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i <= Nq) seq_off[i] = 0;
  if (i < Nq) {
    int p = q_pos[i];
    if (p < 0 || p > max_pos) {
      sa::report(status, sa::kErrDevice, sa::kKernIndexerPrefill, i, p, max_pos);
      p = -1;  // row skipped
    }
    seq_len[i] = p + 1;
  }
}

}  // namespace

extern "C" {

const char* sa_status_string(sa_status s) {
  switch (s) {
    case SA_OK: return "SA_OK";
    case SA_ERR_INVALID_ARG: return "SA_ERR_INVALID_ARG";
    case SA_ERR_UNSUPPORTED: return "SA_ERR_UNSUPPORTED";
    case SA_ERR_WORKSPACE: return "SA_ERR_WORKSPACE";
    case SA_ERR_CUDA: return "SA_ERR_CUDA";
    case SA_ERR_TIMEOUT: return "SA_ERR_TIMEOUT";
    case SA_ERR_DEVICE: return "SA_ERR_DEVICE";
    default: return "SA_ERR_UNKNOWN";
  }
}

const char* sa_last_error(void) { return g_last_error.c_str(); }

int sa_abi_version(void) { return 1; }

sa_status sa_read_device_status(const void* ws, void* stream, int* device_status, int64_t* detail) {
  if (!ws || !device_status) return fail(SA_ERR_INVALID_ARG, "sa_read_device_status: NULL argument");
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail("sa_read_device_status sync", e);
  sa::DeviceStatus st;
  e = cudaMemcpy(&st, ws, sizeof st, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail("sa_read_device_status copy", e);
  *device_status = st.code;
  if (detail)
    for (int i = 0; i < 4; ++i) detail[i] = st.detail[i];
  return SA_OK;
}

sa_status sa_clear_device_status(void* ws, void* stream) {
  if (!ws) return fail(SA_ERR_INVALID_ARG, "sa_clear_device_status: NULL workspace");
  cudaError_t e = cudaMemsetAsync(ws, 0, SA_WS_HEADER_BYTES, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail("sa_clear_device_status", e);
  return SA_OK;
}

}  // extern "C"

namespace {
// One CTA waits on an mbarrier that nothing arrives on: the wait routine of
// every kernel must give up after limit_ns and the give-up must be reported.
__global__ void wait_probe_kernel(sa::DeviceStatus* status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    sa::mbar_init(&bar, 1);
    sa::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !sa::mbar_wait(&bar, 0, limit_ns))
    sa::report(status, sa::kErrTimeout, sa::kKernWaitProbe, 0, 0, (long long)limit_ns);
  __syncthreads();
}
}  // namespace

extern "C" {

sa_status sa_wait_probe(void* ws, size_t ws_bytes, unsigned long long limit_ns, void* stream) {
  const char* who = "sa_wait_probe";
  if (limit_ns < 1000ull || limit_ns > 1000000000ull)
    return fail(SA_ERR_INVALID_ARG, "%s: limit_ns=%llu outside [1e3, 1e9]", who, limit_ns);
  sa_status st = check_ws(ws, ws_bytes, SA_WS_HEADER_BYTES, who);
  if (st != SA_OK) return st;
  wait_probe_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(status_of(ws), limit_ns);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail("sa_wait_probe launch", e);
  return SA_OK;
}

// ---------------------------------------------------------------- indexer
size_t sa_index_score_workspace_size(int B) {
  (void)B;
  return SA_WS_HEADER_BYTES;
}

static sa_status index_score_impl(const void* qI, const float* w, const void* KI, const int64_t* seq_off,
                                  const int32_t* seq_len, int B, int64_t n_tokens, int S_max, int H_I, int d_I,
                                  float* scores, int64_t ld, void* ws, size_t ws_bytes, void* stream,
                                  const sa::AppendArgs& ap, const char* who);

sa_status sa_index_score(const void* qI, const float* w, const void* KI, const int64_t* seq_off,
                         const int32_t* seq_len, int B, int64_t n_tokens, int S_max, int H_I, int d_I, float* scores,
                         int64_t ld, void* ws, size_t ws_bytes, void* stream) {
  return index_score_impl(qI, w, KI, seq_off, seq_len, B, n_tokens, S_max, H_I, d_I, scores, ld, ws, ws_bytes,
                          stream, sa::AppendArgs{}, "sa_index_score");
}

static sa_status index_score_impl(const void* qI, const float* w, const void* KI, const int64_t* seq_off,
                                  const int32_t* seq_len, int B, int64_t n_tokens, int S_max, int H_I, int d_I,
                                  float* scores, int64_t ld, void* ws, size_t ws_bytes, void* stream,
                                  const sa::AppendArgs& ap, const char* who) {
  if (B < 0 || B > 4096) return fail(SA_ERR_INVALID_ARG, "%s: B=%d outside [0, 4096]", who, B);
  if (S_max < 0) return fail(SA_ERR_INVALID_ARG, "%s: S_max=%d < 0", who, S_max);
  if (n_tokens < 1 || n_tokens >= (1ll << 31)) return fail(SA_ERR_INVALID_ARG, "%s: n_tokens=%lld outside [1, 2^31)", who, (long long)n_tokens);
  if (ld < S_max) return fail(SA_ERR_INVALID_ARG, "%s: ld=%lld < S_max=%d", who, (long long)ld, S_max);
  sa_status st = validate_index(qI, w, KI, H_I, d_I, who);
  if (st != SA_OK) return st;
  if (!seq_off || !seq_len || !scores) return fail(SA_ERR_INVALID_ARG, "%s: NULL pointer", who);
  if ((st = check_ws(ws, ws_bytes, sa_index_score_workspace_size(B), who)) != SA_OK) return st;
  if (B == 0 || S_max == 0) return SA_OK;
  return run_index_decode(qI, w, KI, seq_off, seq_len, B, n_tokens, S_max, H_I, d_I, scores, ld, ws,
                          (cudaStream_t)stream, ap);
}

size_t sa_index_score_prefill_workspace_size(int Nq) {
  return SA_WS_HEADER_BYTES + round_up(8 * ((size_t)Nq + 1), 256) + round_up(4 * (size_t)Nq, 256);
}

sa_status sa_index_score_prefill(const void* qI, const float* w, const void* KI, const int32_t* q_pos, int Nq, int S,
                                 int max_pos, int H_I, int d_I, float* scores, int64_t ld, void* ws, size_t ws_bytes,
                                 void* stream) {
  const char* who = "sa_index_score_prefill";
  if (Nq < 0 || Nq > 4096) return fail(SA_ERR_INVALID_ARG, "%s: Nq=%d outside [0, 4096]", who, Nq);
  if (S < 1 || max_pos < 0 || max_pos >= S) return fail(SA_ERR_INVALID_ARG, "%s: need 0 <= max_pos < S", who);
  if (ld < (int64_t)max_pos + 1) return fail(SA_ERR_INVALID_ARG, "%s: ld below max_pos + 1", who);
  sa_status st = validate_index(qI, w, KI, H_I, d_I, who);
  if (st != SA_OK) return st;
  if (!q_pos || !scores) return fail(SA_ERR_INVALID_ARG, "%s: NULL pointer", who);
  if ((st = check_ws(ws, ws_bytes, sa_index_score_prefill_workspace_size(Nq), who)) != SA_OK) return st;
  if (Nq == 0) return SA_OK;
  cudaStream_t s = (cudaStream_t)stream;
  if (sa::indexer_prefill_supported(H_I, d_I)) {
    // blocks of 256 / H_I queries share every key tile on the tensor cores
    CUtensorMap tm_ki, tm_qi;
    const uint64_t kd[2] = {(uint64_t)d_I, (uint64_t)S};
    const uint64_t ks[1] = {(uint64_t)d_I * 2};
    const uint32_t kb[2] = {64, 128};
    if ((st = make_tmap(&tm_ki, KI, 2, kd, ks, kb)) != SA_OK) return st;
    const uint64_t qd[2] = {(uint64_t)d_I, (uint64_t)Nq * H_I};
    const uint64_t qs[1] = {(uint64_t)d_I * 2};
    const uint32_t qb[2] = {64, 256};
    if ((st = make_tmap(&tm_qi, qI, 2, qd, qs, qb)) != SA_OK) return st;
    sa::PrefillIndexerArgs a{w, q_pos, Nq, S, max_pos, H_I, d_I, scores, ld, status_of(ws)};
    cudaError_t e = sa::launch_indexer_prefill(a, tm_ki, tm_qi, num_sms(), s);
    if (e != cudaSuccess) return cuda_fail("sa_index_score_prefill launch", e);
    return SA_OK;
  }
  uint8_t* p = reinterpret_cast<uint8_t*>(ws) + SA_WS_HEADER_BYTES;
  int64_t* soff = reinterpret_cast<int64_t*>(p);
  int32_t* slen = reinterpret_cast<int32_t*>(p + round_up(8 * ((size_t)Nq + 1), 256));
  prefill_rows_kernel<<<(Nq + 256) / 256, 256, 0, s>>>(q_pos, Nq, max_pos, soff, slen, status_of(ws));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail("sa_index_score_prefill rows", e);
  // every query is a row of its own over the one cache: the decode kernel with
  // seq_off = 0 and seq_len = q_pos + 1
  return run_index_decode(qI, w, KI, soff, slen, Nq, S, max_pos + 1, H_I, d_I, scores, ld, ws, s);
}

// ---------------------------------------------------------------- prefill indexer + top-k, blocked
namespace {
// Queries per block: all of them by default.  The indexer streams every key
// tile once per block of queries, so smaller blocks trade time for
// workspace (c4, S = 131072: 1.93 ms for one block of 2048 queries, 3.0 ms
// in blocks of 1024, 5.4 ms of 512, 9.9 ms of 256, 18.9 ms of 128).
int index_topk_rows(int Nq, int S, int rows_per_block) {
  (void)S;
  int nb = rows_per_block > 0 ? rows_per_block : Nq;
  if (nb < 1) nb = 1;
  if (nb > Nq) nb = Nq;
  return nb;
}

struct IndexTopkLayout {
  size_t soff, slen, scores, topk, total;  // byte offsets after the header, then the total
  int rows;
};

IndexTopkLayout index_topk_layout(int Nq, int S, int max_pos, int k, int rows_per_block) {
  IndexTopkLayout l{};
  l.rows = index_topk_rows(Nq, S, rows_per_block);
  l.soff = 0;
  l.slen = round_up(8 * ((size_t)Nq + 1), 256);
  l.scores = l.slen + round_up(4 * (size_t)Nq, 256);
  l.topk = l.scores + round_up((size_t)l.rows * S * 4, 256);
  const size_t t = sa::topk_use_split(l.rows, max_pos + 1, num_sms())
                       ? sa::topk_split_ws_bytes(l.rows, max_pos + 1, num_sms())
                       : 0;
  (void)k;
  l.total = SA_WS_HEADER_BYTES + l.topk + round_up(t, 256);
  return l;
}
}  // namespace

size_t sa_index_topk_prefill_workspace_size(int Nq, int S, int max_pos, int k, int rows_per_block) {
  if (Nq < 1 || S < 1 || max_pos < 0 || max_pos >= S || k < 1) return SA_WS_HEADER_BYTES;
  return index_topk_layout(Nq, S, max_pos, k, rows_per_block).total;
}

sa_status sa_index_topk_prefill(const void* qI, const float* w, const void* KI, const int32_t* q_pos, int Nq, int S,
                                int max_pos, int H_I, int d_I, int k, int rows_per_block, int32_t* idx, void* ws,
                                size_t ws_bytes, void* stream) {
  const char* who = "sa_index_topk_prefill";
  if (Nq < 0 || Nq > 4096) return fail(SA_ERR_INVALID_ARG, "%s: Nq=%d outside [0, 4096]", who, Nq);
  if (S < 1 || max_pos < 0 || max_pos >= S) return fail(SA_ERR_INVALID_ARG, "%s: need 0 <= max_pos < S", who);
  if (k < 1) return fail(SA_ERR_INVALID_ARG, "%s: k=%d < 1", who, k);
  if (rows_per_block < 0) return fail(SA_ERR_INVALID_ARG, "%s: rows_per_block < 0", who);
  sa_status st = validate_index(qI, w, KI, H_I, d_I, who);
  if (st != SA_OK) return st;
  if (!q_pos || !idx) return fail(SA_ERR_INVALID_ARG, "%s: NULL pointer", who);
  if ((st = check_ws(ws, ws_bytes, sa_index_topk_prefill_workspace_size(Nq, S, max_pos, k, rows_per_block), who)) !=
      SA_OK)
    return st;
  if (Nq == 0) return SA_OK;
  cudaStream_t s = (cudaStream_t)stream;
  const IndexTopkLayout l = index_topk_layout(Nq, S, max_pos, k, rows_per_block);
  uint8_t* p = reinterpret_cast<uint8_t*>(ws) + SA_WS_HEADER_BYTES;
  int64_t* soff = reinterpret_cast<int64_t*>(p + l.soff);
  int32_t* slen = reinterpret_cast<int32_t*>(p + l.slen);  // q_pos + 1: each row's valid length
  float* blk = reinterpret_cast<float*>(p + l.scores);
  const int64_t ld = S;
  const int n_max = max_pos + 1;
  prefill_rows_kernel<<<(Nq + 256) / 256, 256, 0, s>>>(q_pos, Nq, max_pos, soff, slen, status_of(ws));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail("sa_index_topk_prefill rows", e);
  const bool tc = sa::indexer_prefill_supported(H_I, d_I);
  CUtensorMap tm_ki;
  if (tc) {
    const uint64_t kd[2] = {(uint64_t)d_I, (uint64_t)S};
    const uint64_t ks[1] = {(uint64_t)d_I * 2};
    const uint32_t kb[2] = {64, 128};
    if ((st = make_tmap(&tm_ki, KI, 2, kd, ks, kb)) != SA_OK) return st;
  }
  // one block of queries at a time: its scores (in the workspace), then its top-k
  for (int j0 = 0; j0 < Nq; j0 += l.rows) {
    const int nb = Nq - j0 < l.rows ? Nq - j0 : l.rows;
    const void* qI_b = reinterpret_cast<const uint8_t*>(qI) + (size_t)j0 * H_I * d_I * 2;
    if (tc) {
      CUtensorMap tm_qi;
      const uint64_t qd[2] = {(uint64_t)d_I, (uint64_t)nb * H_I};
      const uint64_t qs[1] = {(uint64_t)d_I * 2};
      const uint32_t qb[2] = {64, 256};
      if ((st = make_tmap(&tm_qi, qI_b, 2, qd, qs, qb)) != SA_OK) return st;
      sa::PrefillIndexerArgs a{w + (size_t)j0 * H_I, q_pos + j0, nb, S, max_pos, H_I, d_I, blk, ld, status_of(ws)};
      e = sa::launch_indexer_prefill(a, tm_ki, tm_qi, num_sms(), s);
      if (e != cudaSuccess) return cuda_fail("sa_index_topk_prefill indexer launch", e);
    } else {
      st = run_index_decode(qI_b, w + (size_t)j0 * H_I, KI, soff + j0, slen + j0, nb, S, n_max, H_I, d_I, blk, ld, ws,
                            s);
      if (st != SA_OK) return st;
    }
    if (sa::topk_use_split(nb, n_max, num_sms()))
      e = sa::launch_topk_split(blk, ld, slen + j0, nb, n_max, k, idx + (size_t)j0 * k, nullptr, status_of(ws),
                                p + l.topk, num_sms(), s);
    else
      e = sa::launch_topk_rows(blk, ld, slen + j0, nb, n_max, k, idx + (size_t)j0 * k, nullptr, status_of(ws), s);
    if (e != cudaSuccess) return cuda_fail("sa_index_topk_prefill top-k launch", e);
  }
  return SA_OK;
}

// ---------------------------------------------------------------- top-k
size_t sa_topk_workspace_size(int Nq, int n_max, int k) {
  (void)k;
  if (Nq > 0 && n_max > 0 && sa::topk_use_split(Nq, n_max, num_sms()))
    return SA_WS_HEADER_BYTES + sa::topk_split_ws_bytes(Nq, n_max, num_sms());
  return SA_WS_HEADER_BYTES;
}

sa_status sa_topk(const float* scores, int64_t ld, const int32_t* n_valid, int Nq, int n_max, int k, int32_t* idx,
                  float* top_scores, void* ws, size_t ws_bytes, void* stream) {
  const char* who = "sa_topk";
  if (Nq < 0) return fail(SA_ERR_INVALID_ARG, "%s: Nq=%d < 0", who, Nq);
  if (k < 1) return fail(SA_ERR_INVALID_ARG, "%s: k=%d < 1", who, k);
  if (n_max < 0 || ld < n_max) return fail(SA_ERR_INVALID_ARG, "%s: need 0 <= n_max <= ld", who);
  if (Nq > 0 && (!scores || !n_valid || !idx)) return fail(SA_ERR_INVALID_ARG, "%s: NULL pointer", who);
  sa_status st = check_ws(ws, ws_bytes, sa_topk_workspace_size(Nq, n_max, k), who);
  if (st != SA_OK) return st;
  if (Nq == 0) return SA_OK;
  cudaError_t e;
  if (sa::topk_use_split(Nq, n_max, num_sms()))
    e = sa::launch_topk_split(scores, ld, n_valid, Nq, n_max, k, idx, top_scores, status_of(ws),
                              reinterpret_cast<uint8_t*>(ws) + SA_WS_HEADER_BYTES, num_sms(), (cudaStream_t)stream);
  else
    e = sa::launch_topk_rows(scores, ld, n_valid, Nq, n_max, k, idx, top_scores, status_of(ws),
                             (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail("sa_topk launch", e);
  return SA_OK;
}

// ---------------------------------------------------------------- dynamic k
namespace {
struct DynLayout {
  size_t topk, sel_idx, sel_s, total;  // byte offsets after the header, then the total
};
DynLayout dyn_layout(int Nq, int n_max, int k_max) {
  DynLayout l{};
  const size_t t = (Nq > 0 && n_max > 0 && sa::topk_use_split(Nq, n_max, num_sms()))
                       ? sa::topk_split_ws_bytes(Nq, n_max, num_sms())
                       : 0;
  l.topk = 0;
  l.sel_idx = round_up(t, 256);
  l.sel_s = l.sel_idx + round_up(4 * (size_t)Nq * (size_t)k_max, 256);
  l.total = SA_WS_HEADER_BYTES + l.sel_s + round_up(4 * (size_t)Nq * (size_t)k_max, 256);
  return l;
}
}  // namespace

size_t sa_topk_dynamic_workspace_size(int Nq, int n_max, int k_max) {
  if (Nq < 1 || n_max < 1 || k_max < 1) return SA_WS_HEADER_BYTES;
  return dyn_layout(Nq, n_max, k_max).total;
}

sa_status sa_topk_dynamic(const float* scores, int64_t ld, const int32_t* n_valid, int Nq, int n_max, int k_max,
                          double tau, int32_t* idx, int32_t* counts, void* ws, size_t ws_bytes, void* stream) {
  const char* who = "sa_topk_dynamic";
  if (Nq < 0) return fail(SA_ERR_INVALID_ARG, "%s: Nq=%d < 0", who, Nq);
  if (k_max < 1 || k_max > 4096) return fail(SA_ERR_UNSUPPORTED, "%s: k_max=%d outside [1, 4096]", who, k_max);
  if (!(tau > 0.0 && tau <= 1.0)) return fail(SA_ERR_INVALID_ARG, "%s: tau must be in (0, 1]", who);
  if (n_max < 0 || ld < n_max) return fail(SA_ERR_INVALID_ARG, "%s: need 0 <= n_max <= ld", who);
  if (Nq > 0 && (!scores || !n_valid || !idx || !counts)) return fail(SA_ERR_INVALID_ARG, "%s: NULL pointer", who);
  sa_status st = check_ws(ws, ws_bytes, sa_topk_dynamic_workspace_size(Nq, n_max, k_max), who);
  if (st != SA_OK) return st;
  if (Nq == 0) return SA_OK;
  const DynLayout l = dyn_layout(Nq, n_max, k_max);
  uint8_t* base = reinterpret_cast<uint8_t*>(ws) + SA_WS_HEADER_BYTES;
  int32_t* sel_idx = reinterpret_cast<int32_t*>(base + l.sel_idx);
  float* sel_s = reinterpret_cast<float*>(base + l.sel_s);
  const cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e;
  if (sa::topk_use_split(Nq, n_max, num_sms()))
    e = sa::launch_topk_split(scores, ld, n_valid, Nq, n_max, k_max, sel_idx, sel_s, status_of(ws), base + l.topk,
                              num_sms(), s);
  else
    e = sa::launch_topk_rows(scores, ld, n_valid, Nq, n_max, k_max, sel_idx, sel_s, status_of(ws), s);
  if (e != cudaSuccess) return cuda_fail("sa_topk_dynamic top-k launch", e);
  e = sa::launch_topk_dynamic(scores, ld, n_valid, Nq, n_max, sel_idx, sel_s, k_max, tau, idx, counts, status_of(ws),
                              s);
  if (e != cudaSuccess) return cuda_fail("sa_topk_dynamic launch", e);
  return SA_OK;
}

// ---------------------------------------------------------------- attention
// The CUDA-core path (few rows per (b, g)): its per-(b, g) counters sit in the
// workspace header after the status block, the slices' partials after it.
constexpr size_t kSmallCounterOffset = 256;
constexpr int kSmallMaxCounters = (int)((SA_WS_HEADER_BYTES - kSmallCounterOffset) / 4);

bool small_attn_path(int L_g, int Hq, int Hkv) { return (int64_t)L_g * (Hq / Hkv) <= sa::kSmallMaxRows; }

int small_attn_plan(int B, int Hkv, int k) { return sa::small_attn_splits(B * Hkv, k, num_sms(), kSmallMaxCounters); }

// 9 to 128 rows per (b, g) on too few units to fill the GPU (the tcgen05
// plan has fewer CTAs than half the SMs, e.g. one sequence with one KV
// head): the warp-level MMA kernel with one warp per 16 rows, whose key
// slices spread the few units over many CTAs.  With more units the tcgen05
// kernel is faster (c2: 154 against 165 us per step; c3: 63 against 75).
bool mid_attn_path(int L_g, int B, int Hq, int Hkv, int k) {
  const int64_t R = (int64_t)L_g * (Hq / Hkv);
  if (R <= sa::kSmallMaxRows || R > sa::kMidMaxRows) return false;
  if ((int64_t)k > (int64_t)sa::kMidMaxSplits * sa::kMidMaxSlice) return false;
  return plan_decode_attn(L_g, B, Hq, Hkv, k).units * 2 < num_sms();
}

int mid_attn_plan(int B, int Hkv, int R, int k) { return sa::mid_attn_splits(B * Hkv, R, k, num_sms()); }

size_t sa_sparse_decode_attn_workspace_size(int L_g, int B, int Hq, int Hkv, int d, int k) {
  (void)d;
  if (L_g < 1 || B < 1 || Hkv < 1 || Hq < Hkv || k < 1) return SA_WS_HEADER_BYTES;
  if (small_attn_path(L_g, Hq, Hkv))
    return SA_WS_HEADER_BYTES +
           sa::small_attn_scratch_bytes(B * Hkv, small_attn_plan(B, Hkv, k), L_g * (Hq / Hkv));
  if (mid_attn_path(L_g, B, Hq, Hkv, k)) {
    const int R = L_g * (Hq / Hkv);
    const size_t mid = SA_WS_HEADER_BYTES + sa::mid_attn_scratch_bytes(B * Hkv, mid_attn_plan(B, Hkv, R, k), R);
    const size_t big = attn_ws_bytes(plan_decode_attn(L_g, B, Hq, Hkv, k));
    return mid > big ? mid : big;  // the partial-output mode still takes the tcgen05 kernel
  }
  return attn_ws_bytes(plan_decode_attn(L_g, B, Hq, Hkv, k));
}

static sa_status run_decode_attn(const void* Q, const void* K, const void* V, const int64_t* seq_off,
                                 const int32_t* seq_len, const int32_t* idx, int L_g, int B, int64_t n_tokens, int Hq,
                                 int Hkv, int d, int k, float scale, void* O, sa_dtype out_dtype, void* ws,
                                 size_t ws_bytes, cudaStream_t stream, float* ml = nullptr,
                                 const int32_t* idx_count = nullptr, bool early = false) {
  const char* who = ml ? "sa_sparse_decode_attn_partial" : "sa_sparse_decode_attn";
  if (ml && (out_dtype != SA_F32 || !aligned(ml, 8)))
    return fail(SA_ERR_INVALID_ARG, "%s: partial outputs are fp32 and ml 8-byte aligned", who);
  if (L_g < 1 || B < 1 || Hq < 1 || Hkv < 1 || k < 1)
    return fail(SA_ERR_INVALID_ARG, "%s: L_g, B, Hq, Hkv, k must be >= 1", who);
  if (d != 128) return fail(SA_ERR_UNSUPPORTED, "%s: d=%d (only 128 is built)", who, d);
  if (Hq % Hkv != 0) return fail(SA_ERR_INVALID_ARG, "%s: Hq=%d not a multiple of Hkv=%d", who, Hq, Hkv);
  if (out_dtype != SA_BF16 && out_dtype != SA_F32) return fail(SA_ERR_INVALID_ARG, "%s: bad out_dtype", who);
  if (!Q || !K || !V || !seq_off || !seq_len || !idx || !O) return fail(SA_ERR_INVALID_ARG, "%s: NULL pointer", who);
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(O, 16))
    return fail(SA_ERR_INVALID_ARG, "%s: Q, K, V, O must be 16-byte aligned", who);
  if (!(scale > 0.f)) return fail(SA_ERR_INVALID_ARG, "%s: scale must be > 0", who);
  if (!ml && !idx_count && small_attn_path(L_g, Hq, Hkv)) {
    // few query rows per (b, g): the warp-level MMA kernel
    const int ns = small_attn_plan(B, Hkv, k);
    const size_t scratch = sa::small_attn_scratch_bytes(B * Hkv, ns, L_g * (Hq / Hkv));
    sa_status st = check_ws(ws, ws_bytes, SA_WS_HEADER_BYTES + scratch, who);
    if (st != SA_OK) return st;
    sa::AttnArgs a{};
    a.Q = reinterpret_cast<const uint16_t*>(Q);
    a.K = reinterpret_cast<const uint16_t*>(K);
    a.V = reinterpret_cast<const uint16_t*>(V);
    a.seq_off = seq_off;
    a.seq_len = seq_len;
    a.idx = idx;
    a.k = k;
    a.L = L_g;
    a.B = B;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.G = Hq / Hkv;
    a.R = L_g * a.G;
    a.n_split = ns;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.O = O;
    a.out_f32 = out_dtype == SA_F32;
    a.status = status_of(ws);
    a.early = early ? 1 : 0;
    if (ns > 1) {
      uint8_t* base = reinterpret_cast<uint8_t*>(ws);
      const size_t n = (size_t)B * Hkv * ns * sa::small_attn_rows(a.R);
      a.small_cnt = reinterpret_cast<uint32_t*>(base + kSmallCounterOffset);
      a.small_po = reinterpret_cast<float*>(base + SA_WS_HEADER_BYTES);
      a.small_pml = reinterpret_cast<float2*>(base + SA_WS_HEADER_BYTES + round_up(n * 128 * 4, 256));
    }
    cudaError_t e = sa::launch_sparse_attn_small(a, stream);
    if (e != cudaSuccess) return cuda_fail("sa_sparse_decode_attn launch", e);
    return SA_OK;
  }
  if (!ml && !idx_count && mid_attn_path(L_g, B, Hq, Hkv, k)) {
    // 9 to 128 rows per (b, g): the warp-level MMA kernel, one warp per 16 rows
    const int R = L_g * (Hq / Hkv);
    const int ns = mid_attn_plan(B, Hkv, R, k);
    sa_status st = check_ws(ws, ws_bytes, SA_WS_HEADER_BYTES + sa::mid_attn_scratch_bytes(B * Hkv, ns, R), who);
    if (st != SA_OK) return st;
    sa::AttnArgs a{};
    a.Q = reinterpret_cast<const uint16_t*>(Q);
    a.K = reinterpret_cast<const uint16_t*>(K);
    a.V = reinterpret_cast<const uint16_t*>(V);
    a.seq_off = seq_off;
    a.seq_len = seq_len;
    a.idx = idx;
    a.k = k;
    a.L = L_g;
    a.B = B;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.G = Hq / Hkv;
    a.R = R;
    a.n_split = ns;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.O = O;
    a.out_f32 = out_dtype == SA_F32;
    a.status = status_of(ws);
    if (ns > 1) {
      uint8_t* base = reinterpret_cast<uint8_t*>(ws);
      const size_t n = (size_t)B * Hkv * ns * R;
      a.small_po = reinterpret_cast<float*>(base + SA_WS_HEADER_BYTES);
      a.small_pml = reinterpret_cast<float2*>(base + SA_WS_HEADER_BYTES + round_up(n * 128 * 4, 256));
    }
    cudaError_t e = sa::launch_sparse_attn_mid(a, stream);
    if (e != cudaSuccess) return cuda_fail("sa_sparse_decode_attn launch", e);
    return SA_OK;
  }
  const AttnPlan p = plan_decode_attn(L_g, B, Hq, Hkv, k);
  sa_status st = check_ws(ws, ws_bytes, attn_ws_bytes(p), who);
  if (st != SA_OK) return st;
  CUtensorMap tm_q, tm_k, tm_v;
  if ((st = make_rows_tmap(&tm_q, Q, (int64_t)L_g * B * Hq)) != SA_OK) return st;
  if ((st = make_rows_tmap(&tm_k, K, n_tokens * Hkv)) != SA_OK) return st;
  if ((st = make_rows_tmap(&tm_v, V, n_tokens * Hkv)) != SA_OK) return st;
  sa::AttnArgs a{};
  a.Q = reinterpret_cast<const uint16_t*>(Q);
  a.K = reinterpret_cast<const uint16_t*>(K);
  a.V = reinterpret_cast<const uint16_t*>(V);
  a.seq_off = seq_off;
  a.seq_len = seq_len;
  a.idx = idx;
  a.k = k;
  a.prefill = 0;
  a.L = L_g;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.G = Hq / Hkv;
  a.R = L_g * a.G;
  a.n_mtiles = p.n_mtiles;
  a.n_split = p.n_split;
  a.keys_per_split = p.keys_per_split;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.O = O;
  a.out_f32 = out_dtype == SA_F32;
  a.ml = reinterpret_cast<float2*>(ml);
  a.idx_count = idx_count;
  a.status = status_of(ws);
  cudaError_t e = sa::launch_sparse_attn(a, tm_q, tm_k, tm_v, out_dtype == SA_F32, stream);
  if (e != cudaSuccess) return cuda_fail("sa_sparse_decode_attn launch", e);
  return SA_OK;
}

sa_status sa_sparse_decode_attn(const void* Q, const void* K, const void* V, const int64_t* seq_off,
                                const int32_t* seq_len, const int32_t* idx, int L_g, int B, int64_t n_tokens, int Hq,
                                int Hkv, int d, int k, float scale, void* O, sa_dtype out_dtype, void* ws,
                                size_t ws_bytes, void* stream) {
  return run_decode_attn(Q, K, V, seq_off, seq_len, idx, L_g, B, n_tokens, Hq, Hkv, d, k, scale, O, out_dtype, ws,
                         ws_bytes, (cudaStream_t)stream);
}

// ---------------------------------------------------------------- indexer layer (CLSA routing)
size_t sa_indexer_layer_attn_workspace_size(int B, int S_max, int Hq, int Hkv, int d) {
  (void)Hkv;
  (void)d;
  if (B < 1 || S_max < 1 || Hq < 1) return SA_WS_HEADER_BYTES;
  return SA_WS_HEADER_BYTES + sa::route_ws_bytes(B, S_max, Hq);
}

sa_status sa_indexer_layer_attn(const void* Q, const void* K, const void* V, const int64_t* seq_off,
                                const int32_t* seq_len, int B, int64_t n_tokens, int S_max, int Hq, int Hkv, int d,
                                float scale, void* O, sa_dtype out_dtype, float* scores, int64_t ld, void* ws,
                                size_t ws_bytes, void* stream) {
  const char* who = "sa_indexer_layer_attn";
  if (B < 0 || S_max < 0 || n_tokens < 0) return fail(SA_ERR_INVALID_ARG, "%s: negative size", who);
  if (Hq < 1 || Hkv < 1 || Hq % Hkv != 0)
    return fail(SA_ERR_INVALID_ARG, "%s: Hq=%d must be a positive multiple of Hkv=%d", who, Hq, Hkv);
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8)
    return fail(SA_ERR_UNSUPPORTED, "%s: Hq/Hkv=%d not in {1, 2, 4, 8}", who, G);
  if (Hq > 256) return fail(SA_ERR_UNSUPPORTED, "%s: Hq=%d above 256", who, Hq);
  if (d != 128) return fail(SA_ERR_UNSUPPORTED, "%s: d=%d (only 128 is built)", who, d);
  if (out_dtype != SA_BF16 && out_dtype != SA_F32) return fail(SA_ERR_INVALID_ARG, "%s: bad out_dtype", who);
  if (ld < S_max) return fail(SA_ERR_INVALID_ARG, "%s: ld=%lld below S_max=%d", who, (long long)ld, S_max);
  sa_status st = check_ws(ws, ws_bytes, sa_indexer_layer_attn_workspace_size(B, S_max, Hq, Hkv, d), who);
  if (st != SA_OK) return st;
  if (B == 0 || S_max == 0) return SA_OK;
  if (!Q || !K || !V || !seq_off || !seq_len || !O || !scores)
    return fail(SA_ERR_INVALID_ARG, "%s: NULL pointer", who);
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(O, 16) || !aligned(scores, 4))
    return fail(SA_ERR_INVALID_ARG, "%s: Q, K, V, O must be 16-byte aligned and scores 4-byte aligned", who);
  sa::RouteArgs a{};
  a.Q = reinterpret_cast<const uint16_t*>(Q);
  a.K = reinterpret_cast<const uint16_t*>(K);
  a.V = reinterpret_cast<const uint16_t*>(V);
  a.seq_off = seq_off;
  a.seq_len = seq_len;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.S_max = S_max;
  a.n_tokens = n_tokens;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.n_split = (S_max + sa::kRouteChunk - 1) / sa::kRouteChunk;
  a.zld = (int64_t)round_up((size_t)S_max, 64);
  uint8_t* p = reinterpret_cast<uint8_t*>(ws) + SA_WS_HEADER_BYTES;
  a.z = reinterpret_cast<float*>(p);
  p += round_up((size_t)B * Hq * a.zld * 4, 256);
  a.part_ml = reinterpret_cast<float2*>(p);
  p += round_up((size_t)B * Hq * a.n_split * 8, 256);
  a.part_o = reinterpret_cast<float*>(p);
  a.scores = scores;
  a.ld = ld;
  a.O = O;
  a.out_f32 = out_dtype == SA_F32;
  a.status = status_of(ws);
  CUtensorMap tm_k, tm_v, tm_q;
  if ((st = make_tile128_tmap(&tm_k, K, n_tokens * Hkv)) != SA_OK) return st;
  if ((st = make_tile128_tmap(&tm_v, V, n_tokens * Hkv)) != SA_OK) return st;
  {
    const uint64_t dims[3] = {128, (uint64_t)Hq, (uint64_t)B};
    const uint64_t str[2] = {256, (uint64_t)Hq * 256};
    const uint32_t box[3] = {64, 16, 1};
    if ((st = make_tmap(&tm_q, Q, 3, dims, str, box)) != SA_OK) return st;
  }
  const cudaError_t e = sa::launch_indexer_layer_attn(a, tm_k, tm_v, tm_q, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail("sa_indexer_layer_attn launch", e);
  return SA_OK;
}

sa_status sa_sparse_decode_attn_partial(const void* Q, const void* K, const void* V, const int64_t* seq_off,
                                        const int32_t* seq_len, const int32_t* idx, int L_g, int B, int64_t n_tokens,
                                        int Hq, int Hkv, int d, int k, const int32_t* idx_count, float scale,
                                        float* O_part, float* ml, void* ws, size_t ws_bytes, void* stream) {
  if (!ml) return fail(SA_ERR_INVALID_ARG, "sa_sparse_decode_attn_partial: NULL ml");
  return run_decode_attn(Q, K, V, seq_off, seq_len, idx, L_g, B, n_tokens, Hq, Hkv, d, k, scale, O_part, SA_F32, ws,
                         ws_bytes, (cudaStream_t)stream, ml, idx_count);
}

// ---------------------------------------------------------------- context-parallel decode
namespace {
struct CpSelectLayout {
  size_t rows, n_valid, sel, topk, total;  // byte offsets after the header, then the total
};
CpSelectLayout cp_select_layout(int N, int B, int k) {
  CpSelectLayout l{};
  const size_t n = (size_t)N * k;
  l.rows = 0;
  l.n_valid = l.rows + round_up(4 * (size_t)B * n, 256);
  l.sel = l.n_valid + round_up(4 * (size_t)B, 256);
  l.topk = l.sel + round_up(4 * (size_t)B * k, 256);
  const size_t t = sa::topk_use_split(B, (int)n, num_sms()) ? sa::topk_split_ws_bytes(B, (int)n, num_sms()) : 0;
  l.total = SA_WS_HEADER_BYTES + l.topk + round_up(t, 256);
  return l;
}
}  // namespace

size_t sa_cp_select_workspace_size(int N, int B, int k) {
  if (N < 1 || B < 1 || k < 1 || (int64_t)N * k > INT32_MAX) return SA_WS_HEADER_BYTES;
  return cp_select_layout(N, B, k).total;
}

sa_status sa_cp_select(const float* cand_scores, const int32_t* cand_idx, int64_t cand_stride, int N, int B, int k,
                       int rank, int32_t* local_idx, int32_t* local_count, void* ws, size_t ws_bytes, void* stream) {
  const char* who = "sa_cp_select";
  if (N < 1 || B < 1 || k < 1) return fail(SA_ERR_INVALID_ARG, "%s: N, B, k must be >= 1", who);
  if ((int64_t)N * k > INT32_MAX) return fail(SA_ERR_INVALID_ARG, "%s: N*k above 2^31 - 1", who);
  if (rank < 0 || rank >= N) return fail(SA_ERR_INVALID_ARG, "%s: rank=%d outside [0, %d)", who, rank, N);
  if (!cand_scores || !cand_idx || !local_idx) return fail(SA_ERR_INVALID_ARG, "%s: NULL pointer", who);
  if (N > 1 && cand_stride < (int64_t)B * k)
    return fail(SA_ERR_INVALID_ARG, "%s: cand_stride=%lld below B*k", who, (long long)cand_stride);
  sa_status st = check_ws(ws, ws_bytes, sa_cp_select_workspace_size(N, B, k), who);
  if (st != SA_OK) return st;
  const CpSelectLayout l = cp_select_layout(N, B, k);
  uint8_t* base = reinterpret_cast<uint8_t*>(ws) + SA_WS_HEADER_BYTES;
  float* rows = reinterpret_cast<float*>(base + l.rows);
  int32_t* n_valid = reinterpret_cast<int32_t*>(base + l.n_valid);
  int32_t* sel = reinterpret_cast<int32_t*>(base + l.sel);
  const cudaStream_t s = (cudaStream_t)stream;
  const int n = N * k;
  cudaError_t e = sa::launch_cp_gather(cand_scores, cand_idx, cand_stride, N, B, k, rows, n_valid, s);
  if (e != cudaSuccess) return cuda_fail("sa_cp_select gather launch", e);
  if (sa::topk_use_split(B, n, num_sms()))
    e = sa::launch_topk_split(rows, n, n_valid, B, n, k, sel, nullptr, status_of(ws), base + l.topk, num_sms(), s);
  else
    e = sa::launch_topk_rows(rows, n, n_valid, B, n, k, sel, nullptr, status_of(ws), s);
  if (e != cudaSuccess) return cuda_fail("sa_cp_select top-k launch", e);
  e = sa::launch_cp_local(sel, cand_idx, cand_stride, B, k, rank, local_idx, local_count, s);
  if (e != cudaSuccess) return cuda_fail("sa_cp_select local launch", e);
  return SA_OK;
}

size_t sa_cp_radix_workspace_size(int B) {
  if (B < 1) return SA_WS_HEADER_BYTES;
  return SA_WS_HEADER_BYTES + round_up((size_t)B * sizeof(sa::CpRadixState), 256);
}

static sa_status cp_radix_check(const float* scores, int64_t ld, const int32_t* n_local, int B, int k, int N,
                                int level, const int32_t* gathered, int64_t rank_stride, void* ws, size_t ws_bytes,
                                const char* who) {
  if (B < 1 || k < 1 || N < 1) return fail(SA_ERR_INVALID_ARG, "%s: B, k, N must be >= 1", who);
  if (N > 1024) return fail(SA_ERR_UNSUPPORTED, "%s: N=%d above 1024 ranks", who, N);
  if (!scores || !n_local) return fail(SA_ERR_INVALID_ARG, "%s: NULL pointer", who);
  if (ld < 1) return fail(SA_ERR_INVALID_ARG, "%s: ld must be >= 1", who);
  if (level > 0) {
    const int64_t prev = level == 3 ? 256 : 4096;  // bins of the level whose histograms are gathered
    if (!gathered) return fail(SA_ERR_INVALID_ARG, "%s: NULL gathered histograms", who);
    if (N > 1 && rank_stride < (int64_t)B * prev)
      return fail(SA_ERR_INVALID_ARG, "%s: rank_stride=%lld below B*%lld", who, (long long)rank_stride,
                  (long long)prev);
  }
  return check_ws(ws, ws_bytes, sa_cp_radix_workspace_size(B), who);
}

sa_status sa_cp_radix_level(const float* scores, int64_t ld, const int32_t* n_local, int B, int k, int N, int level,
                            const int32_t* gathered, int64_t rank_stride, int32_t* hist_out, void* ws,
                            size_t ws_bytes, void* stream) {
  const char* who = "sa_cp_radix_level";
  if (level < 0 || level > 2) return fail(SA_ERR_INVALID_ARG, "%s: level=%d outside [0, 2]", who, level);
  if (!hist_out) return fail(SA_ERR_INVALID_ARG, "%s: NULL hist_out", who);
  sa_status st = cp_radix_check(scores, ld, n_local, B, k, N, level, gathered, rank_stride, ws, ws_bytes, who);
  if (st != SA_OK) return st;
  auto* state = reinterpret_cast<sa::CpRadixState*>(reinterpret_cast<uint8_t*>(ws) + SA_WS_HEADER_BYTES);
  cudaError_t e = sa::launch_cp_radix_level(scores, ld, n_local, B, k, N, level, gathered, rank_stride, state,
                                            hist_out, status_of(ws), (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail("sa_cp_radix_level launch", e);
  return SA_OK;
}

sa_status sa_cp_radix_select(const float* scores, int64_t ld, const int32_t* n_local, int B, int k, int N, int rank,
                             const int32_t* gathered, int64_t rank_stride, int32_t* local_idx, int32_t* local_count,
                             void* ws, size_t ws_bytes, void* stream) {
  const char* who = "sa_cp_radix_select";
  if (N >= 1 && (rank < 0 || rank >= N)) return fail(SA_ERR_INVALID_ARG, "%s: rank=%d outside [0, %d)", who, rank, N);
  if (!local_idx) return fail(SA_ERR_INVALID_ARG, "%s: NULL local_idx", who);
  sa_status st = cp_radix_check(scores, ld, n_local, B, k, N, 3, gathered, rank_stride, ws, ws_bytes, who);
  if (st != SA_OK) return st;
  auto* state = reinterpret_cast<const sa::CpRadixState*>(reinterpret_cast<uint8_t*>(ws) + SA_WS_HEADER_BYTES);
  cudaError_t e = sa::launch_cp_radix_finish(scores, ld, n_local, B, k, N, rank, gathered, rank_stride, state,
                                             local_idx, local_count, status_of(ws), (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail("sa_cp_radix_select launch", e);
  return SA_OK;
}

sa_status sa_combine_partials(const float* O_part, int64_t o_stride, const float* ml, int64_t ml_stride, int P,
                              int64_t rows, int d, void* O, sa_dtype out_dtype, void* stream) {
  const char* who = "sa_combine_partials";
  if (P < 1 || rows < 0) return fail(SA_ERR_INVALID_ARG, "%s: need P >= 1, rows >= 0", who);
  if (d != 128) return fail(SA_ERR_UNSUPPORTED, "%s: d=%d (only 128 is built)", who, d);
  if (out_dtype != SA_BF16 && out_dtype != SA_F32) return fail(SA_ERR_INVALID_ARG, "%s: bad out_dtype", who);
  if (rows == 0) return SA_OK;
  if (!O_part || !ml || !O) return fail(SA_ERR_INVALID_ARG, "%s: NULL pointer", who);
  if (!aligned(O_part, 16) || !aligned(ml, 8) || !aligned(O, 16))
    return fail(SA_ERR_INVALID_ARG, "%s: O_part and O must be 16-byte aligned, ml 8-byte aligned", who);
  if (P > 1 && (o_stride < rows * d || o_stride % 4 != 0 || ml_stride < 2 * rows || ml_stride % 2 != 0))
    return fail(SA_ERR_INVALID_ARG, "%s: need o_stride >= rows*d, a multiple of 4, and ml_stride >= 2*rows, even",
                who);
  cudaError_t e = sa::launch_combine_partials(O_part, o_stride, reinterpret_cast<const float2*>(ml), ml_stride / 2, P,
                                              rows, O, out_dtype == SA_F32, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail("sa_combine_partials launch", e);
  return SA_OK;
}

// ---------------------------------------------------------------- decode step
size_t sa_decode_step_workspace_size(int n_layers, int B, int S_max, int Hq, int Hkv, int d, int k) {
  size_t need = SA_WS_HEADER_BYTES;
  // the largest fused group is the whole pattern
  for (int L = 1; L <= n_layers; ++L) {
    const size_t a = sa_sparse_decode_attn_workspace_size(L, B, Hq, Hkv, d, k);
    if (a > need) need = a;
  }
  const size_t t = sa_topk_workspace_size(B, S_max, k);
  return t > need ? t : need;
}

sa_status sa_decode_step(const char* pattern, int n_layers, const void* const* qI, const float* const* w,
                         const void* const* KI, const void* const* K, const void* const* V, const int64_t* seq_off,
                         const int32_t* seq_len, int B, int64_t n_tokens, int S_max, int H_I, int d_I, int k,
                         const void* Q, int Hq, int Hkv, int d, float scale, void* O, sa_dtype out_dtype, int32_t* idx,
                         float* scores, int64_t ld, void* ws, size_t ws_bytes, void* stream) {
  return sa_decode_step_ex(pattern, n_layers, qI, w, const_cast<void* const*>(KI), const_cast<void* const*>(K),
                           const_cast<void* const*>(V), nullptr, nullptr, nullptr, seq_off, seq_len, B, n_tokens,
                           S_max, H_I, d_I, k, Q, Hq, Hkv, d, scale, O, out_dtype, idx, scores, ld, 0, ws, ws_bytes,
                           stream);
}

sa_status sa_decode_step_ex(const char* pattern, int n_layers, const void* const* qI, const float* const* w,
                            void* const* KI, void* const* K, void* const* V, const void* const* new_KI,
                            const void* const* new_K, const void* const* new_V, const int64_t* seq_off,
                            const int32_t* seq_len, int B, int64_t n_tokens, int S_max, int H_I, int d_I, int k,
                            const void* Q, int Hq, int Hkv, int d, float scale, void* O, sa_dtype out_dtype,
                            int32_t* idx, float* scores, int64_t ld, int flags, void* ws, size_t ws_bytes,
                            void* stream) {
  const char* who = "sa_decode_step";
  if (!pattern || n_layers < 1) return fail(SA_ERR_INVALID_ARG, "%s: empty layer pattern", who);
  if ((int)strnlen(pattern, (size_t)n_layers + 1) < n_layers)
    return fail(SA_ERR_INVALID_ARG, "%s: pattern shorter than n_layers", who);
  if (pattern[0] != 'F')
    return fail(SA_ERR_INVALID_ARG, "%s: the first layer must be F (an S layer reuses an upstream F index)", who);
  for (int l = 0; l < n_layers; ++l)
    if (pattern[l] != 'F' && pattern[l] != 'S') return fail(SA_ERR_INVALID_ARG, "%s: pattern letters are F or S", who);
  if (!qI || !w || !KI || !K || !V) return fail(SA_ERR_INVALID_ARG, "%s: NULL pointer array", who);
  if (B < 1 || !Q || !O || !idx || !scores) return fail(SA_ERR_INVALID_ARG, "%s: NULL pointer or B < 1", who);
  if (flags & ~SA_STEP_PER_LAYER) return fail(SA_ERR_INVALID_ARG, "%s: unknown flags 0x%x", who, flags);
  if ((new_K == nullptr) != (new_V == nullptr))
    return fail(SA_ERR_INVALID_ARG, "%s: new_K and new_V come together", who);
  if (new_K && !new_KI) return fail(SA_ERR_INVALID_ARG, "%s: a K/V append needs new_KI too", who);
  if (new_KI) {
    int f = 0;
    for (int l = 0; l < n_layers; ++l) {
      if (pattern[l] == 'F') {
        f = l;
        if (!new_KI[l] || !aligned(new_KI[l], 16) || (new_K && (!new_K[l] || !new_V[l] || !aligned(new_K[l], 16) ||
                                                                !aligned(new_V[l], 16))))
          return fail(SA_ERR_INVALID_ARG, "%s: layer %d: new rows must be non-NULL and 16-byte aligned", who, l);
      } else if (new_K && (K[l] != K[f] || V[l] != V[f])) {
        return fail(SA_ERR_UNSUPPORTED, "%s: appending needs every layer to read its F layer's KV cache (layer %d)",
                    who, l);
      }
    }
  }
  sa_status st = check_ws(ws, ws_bytes, sa_decode_step_workspace_size(n_layers, B, S_max, Hq, Hkv, d, k), who);
  if (st != SA_OK) return st;
  const size_t esize = out_dtype == SA_F32 ? 4 : 2;
  const size_t layer_elems = (size_t)B * Hq * d;
  int l = 0;
  bool prev_small = false;  // the previous launch of this call was the few-rows attention kernel
  while (l < n_layers) {
    if (pattern[l] == 'F') {
      prev_small = false;
      sa::AppendArgs ap{};
      if (new_KI) {
        ap.qI = static_cast<const uint16_t*>(qI[l]);
        ap.new_KI = static_cast<const uint16_t*>(new_KI[l]);
        ap.KI = static_cast<uint16_t*>(KI[l]);
        if (new_K) {
          ap.new_K = static_cast<const uint16_t*>(new_K[l]);
          ap.new_V = static_cast<const uint16_t*>(new_V[l]);
          ap.K = static_cast<uint16_t*>(K[l]);
          ap.V = static_cast<uint16_t*>(V[l]);
        }
        ap.Hkv = Hkv;
        ap.d = d;
      }
      st = index_score_impl(qI[l], w[l], KI[l], seq_off, seq_len, B, n_tokens, S_max, H_I, d_I, scores, ld, ws,
                            ws_bytes, stream, ap, who);
      if (st != SA_OK) return st;
      st = sa_topk(scores, ld, seq_len, B, S_max, k, idx, nullptr, ws, ws_bytes, stream);
      if (st != SA_OK) return st;
    }
    // fuse the following S layers that read the same cache into one group
    // call, unless each layer is to run on its own
    int m = l;
    if (!(flags & SA_STEP_PER_LAYER))
      while (m + 1 < n_layers && pattern[m + 1] == 'S' && K[m + 1] == K[l] && V[m + 1] == V[l]) ++m;
    // after another launch of the few-rows kernel (which writes neither the
    // index nor the caches), this one may start its loads before the wait
    const bool small = small_attn_path(m - l + 1, Hq, Hkv);
    st = run_decode_attn(reinterpret_cast<const uint8_t*>(Q) + (size_t)l * layer_elems * 2, K[l], V[l], seq_off,
                         seq_len, idx, m - l + 1, B, n_tokens, Hq, Hkv, d, k, scale,
                         reinterpret_cast<uint8_t*>(O) + (size_t)l * layer_elems * esize, out_dtype, ws, ws_bytes,
                         (cudaStream_t)stream, nullptr, nullptr, prev_small && small);
    if (st != SA_OK) return st;
    prev_small = small;
    l = m + 1;
  }
  return SA_OK;
}

// ---------------------------------------------------------------- prefill union
}  // extern "C"

// Paged causal attention of a prefill chunk over the group tables
// (kv_indptr, kv_indices) written by the union kernels, or, with osk_order,
// over each row tile's ordered list with ordered skipping (one CTA per row
// tile, no key splits).
static sa_status prefill_attn(const void* Q, const void* K, const void* V, const int32_t* q_pos,
                              const int32_t* kv_indptr, const int32_t* kv_indices, int S, int Nq, int Hq, int Hkv,
                              int block, float scale, void* O, sa_dtype out_dtype, sa::DeviceStatus* status,
                              const int32_t* osk_order, int64_t osk_ld, float osk_tau, int32_t* osk_steps,
                              cudaStream_t s, const char* who) {
  sa::AttnArgs a{};
  a.Q = reinterpret_cast<const uint16_t*>(Q);
  a.K = reinterpret_cast<const uint16_t*>(K);
  a.V = reinterpret_cast<const uint16_t*>(V);
  a.prefill = 1;
  a.q_pos = q_pos;
  a.kv_indptr = kv_indptr;
  a.kv_indices = kv_indices;
  a.S = S;
  a.block = block;
  a.Nq = Nq;
  a.L = 1;
  a.B = 1;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.G = Hq / Hkv;
  a.R = Nq * a.G;
  a.n_mtiles = (a.R + 127) / 128;
  a.n_split = osk_order != nullptr ? 1 : prefill_split(Hkv * a.n_mtiles);
  a.keys_per_split = (int)round_up((size_t)((S + block - 1) / block) * block, 128);
  a.scale_log2 = scale * 1.4426950408889634f;
  a.O = O;
  a.out_f32 = out_dtype == SA_F32;
  a.status = status;
  a.osk_order = osk_order;
  a.osk_ld = osk_ld;
  a.osk_tau = osk_tau;
  a.osk_steps = osk_steps;
  CUtensorMap tm_q, tm_k, tm_v;
  sa_status st2;
  if ((st2 = make_rows_tmap(&tm_q, Q, (int64_t)Nq * Hq)) != SA_OK) return st2;
  if ((st2 = make_block_tmap(&tm_k, K, (int64_t)Hkv * S)) != SA_OK) return st2;
  if ((st2 = make_block_tmap(&tm_v, V, (int64_t)Hkv * S)) != SA_OK) return st2;
  const cudaError_t e = sa::launch_sparse_attn(a, tm_q, tm_k, tm_v, out_dtype == SA_F32, s);
  if (e != cudaSuccess) return cuda_fail(who, e);
  return SA_OK;
}

extern "C" {

size_t sa_block_union_prefill_workspace_size(int S, int Nq, int Hq, int Hkv, int d, int k, int block) {
  (void)Nq;
  (void)Hq;
  (void)Hkv;
  (void)d;
  (void)k;
  if (S < 1 || block < 1) return SA_WS_HEADER_BYTES;
  return SA_WS_HEADER_BYTES + round_up((size_t)(S + block - 1) / block, 256);
}

sa_status sa_block_union_prefill(const int32_t* idx, const int32_t* q_pos, const void* Q, const void* K, const void* V,
                                 int S, int Nq, int Hq, int Hkv, int d, int k, int block, float scale,
                                 int32_t* kv_indptr, int32_t* kv_indices, void* O, sa_dtype out_dtype, void* ws,
                                 size_t ws_bytes, void* stream) {
  const char* who = "sa_block_union_prefill";
  if (S < 1 || Nq < 1 || Hq < 1 || Hkv < 1 || k < 1) return fail(SA_ERR_INVALID_ARG, "%s: sizes must be >= 1", who);
  if (d != 128) return fail(SA_ERR_UNSUPPORTED, "%s: d=%d (only 128 is built)", who, d);
  if (block != 64) return fail(SA_ERR_UNSUPPORTED, "%s: block=%d (only 64 is built)", who, block);
  if (Hq % Hkv != 0) return fail(SA_ERR_INVALID_ARG, "%s: Hq not a multiple of Hkv", who);
  if ((int64_t)Nq * (Hq / Hkv) > (1 << 30)) return fail(SA_ERR_INVALID_ARG, "%s: too many query rows", who);
  if (out_dtype != SA_BF16 && out_dtype != SA_F32) return fail(SA_ERR_INVALID_ARG, "%s: bad out_dtype", who);
  if (!idx || !q_pos || !Q || !K || !V || !kv_indptr || !kv_indices || !O)
    return fail(SA_ERR_INVALID_ARG, "%s: NULL pointer", who);
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(O, 16))
    return fail(SA_ERR_INVALID_ARG, "%s: Q, K, V, O must be 16-byte aligned", who);
  if (!(scale > 0.f)) return fail(SA_ERR_INVALID_ARG, "%s: scale must be > 0", who);
  sa_status st = check_ws(ws, ws_bytes, sa_block_union_prefill_workspace_size(S, Nq, Hq, Hkv, d, k, block), who);
  if (st != SA_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  uint8_t* mark = reinterpret_cast<uint8_t*>(ws) + SA_WS_HEADER_BYTES;
  cudaError_t e = sa::launch_block_union(idx, Nq, k, S, block, Hkv, mark, kv_indptr, kv_indices, status_of(ws), s);
  if (e != cudaSuccess) return cuda_fail("sa_block_union_prefill union", e);
  return prefill_attn(Q, K, V, q_pos, kv_indptr, kv_indices, S, Nq, Hq, Hkv, block, scale, O, out_dtype,
                      status_of(ws), nullptr, 0, 0.f, nullptr, s, "sa_block_union_prefill attention");
}

// ---------------------------------------------------------------- ordered skipping
size_t sa_kap_order_workspace_size(void) { return SA_WS_HEADER_BYTES; }

sa_status sa_kap_order(const int32_t* idx, int Nq, int k, int S, int block, int q_block, const int32_t* kv_indptr,
                       const int32_t* kv_indices, int32_t* order, int64_t ld, void* ws, size_t ws_bytes,
                       void* stream) {
  const char* who = "sa_kap_order";
  if (Nq < 1 || k < 1 || S < 1 || block < 1 || q_block < 1) return fail(SA_ERR_INVALID_ARG, "%s: sizes must be >= 1", who);
  const int64_t nb = ((int64_t)S + block - 1) / block;
  if (nb > sa::kKapMaxBlocks)
    return fail(SA_ERR_UNSUPPORTED, "%s: %lld KV blocks (at most %d are built)", who, (long long)nb, sa::kKapMaxBlocks);
  if (ld < nb) return fail(SA_ERR_INVALID_ARG, "%s: ld=%lld is below ceil(S/block)=%lld", who, (long long)ld, (long long)nb);
  if (!idx || !kv_indptr || !kv_indices || !order) return fail(SA_ERR_INVALID_ARG, "%s: NULL pointer", who);
  sa_status st = check_ws(ws, ws_bytes, sa_kap_order_workspace_size(), who);
  if (st != SA_OK) return st;
  cudaError_t e = sa::launch_kap_order(idx, Nq, k, S, block, q_block, kv_indptr, kv_indices, order, ld,
                                       status_of(ws), (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(who, e);
  return SA_OK;
}

size_t sa_osk_prefill_workspace_size(int S, int Nq, int Hq, int Hkv, int d, int k, int block) {
  return sa_block_union_prefill_workspace_size(S, Nq, Hq, Hkv, d, k, block);
}

sa_status sa_osk_prefill(const int32_t* idx, const int32_t* q_pos, const void* Q, const void* K, const void* V, int S,
                         int Nq, int Hq, int Hkv, int d, int k, int block, float scale, float tau, int32_t* kv_indptr,
                         int32_t* kv_indices, int32_t* order, int32_t* steps, void* O, sa_dtype out_dtype, void* ws,
                         size_t ws_bytes, void* stream) {
  const char* who = "sa_osk_prefill";
  if (S < 1 || Nq < 1 || Hq < 1 || Hkv < 1 || k < 1) return fail(SA_ERR_INVALID_ARG, "%s: sizes must be >= 1", who);
  if (d != 128) return fail(SA_ERR_UNSUPPORTED, "%s: d=%d (only 128 is built)", who, d);
  if (block != 64) return fail(SA_ERR_UNSUPPORTED, "%s: block=%d (only 64 is built)", who, block);
  if (Hq % Hkv != 0) return fail(SA_ERR_INVALID_ARG, "%s: Hq not a multiple of Hkv", who);
  const int G = Hq / Hkv;
  if (128 % G != 0) return fail(SA_ERR_UNSUPPORTED, "%s: Hq/Hkv=%d does not divide 128", who, G);
  if ((int64_t)Nq * G > (1 << 30)) return fail(SA_ERR_INVALID_ARG, "%s: too many query rows", who);
  const int64_t nb = ((int64_t)S + block - 1) / block;
  if (nb > sa::kKapMaxBlocks)
    return fail(SA_ERR_UNSUPPORTED, "%s: %lld KV blocks (at most %d are built)", who, (long long)nb, sa::kKapMaxBlocks);
  if (out_dtype != SA_BF16 && out_dtype != SA_F32) return fail(SA_ERR_INVALID_ARG, "%s: bad out_dtype", who);
  if (!idx || !q_pos || !Q || !K || !V || !kv_indptr || !kv_indices || !order || !steps || !O)
    return fail(SA_ERR_INVALID_ARG, "%s: NULL pointer", who);
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(O, 16))
    return fail(SA_ERR_INVALID_ARG, "%s: Q, K, V, O must be 16-byte aligned", who);
  if (!(scale > 0.f)) return fail(SA_ERR_INVALID_ARG, "%s: scale must be > 0", who);
  if (!(tau >= 0.f) || tau > 3.0e38f) return fail(SA_ERR_INVALID_ARG, "%s: tau must be finite and >= 0", who);
  sa_status st = check_ws(ws, ws_bytes, sa_osk_prefill_workspace_size(S, Nq, Hq, Hkv, d, k, block), who);
  if (st != SA_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  uint8_t* mark = reinterpret_cast<uint8_t*>(ws) + SA_WS_HEADER_BYTES;
  cudaError_t e = sa::launch_block_union(idx, Nq, k, S, block, Hkv, mark, kv_indptr, kv_indices, status_of(ws), s);
  if (e != cudaSuccess) return cuda_fail("sa_osk_prefill union", e);
  e = sa::launch_kap_order(idx, Nq, k, S, block, 128 / G, kv_indptr, kv_indices, order, nb, status_of(ws), s);
  if (e != cudaSuccess) return cuda_fail("sa_osk_prefill order", e);
  return prefill_attn(Q, K, V, q_pos, kv_indptr, kv_indices, S, Nq, Hq, Hkv, block, scale, O, out_dtype,
                      status_of(ws), order, nb, tau, steps, s, "sa_osk_prefill attention");
}

}  // extern "C"

// ---------------------------------------------------------------- no-alloc variant
// Scratch of sa_block_union_prefill_noalloc: a status block followed by one
// byte per KV block.  It lives in the library's own device memory (every GPU
// that loads libsa keeps these bytes until the process exits), so the caller
// needs no workspace.  All calls on a device share it.
#define SA_NOALLOC_MARK_BYTES SA_NOALLOC_MAX_KV_BLOCKS
static __device__ __align__(256) uint8_t g_noalloc_scratch[SA_WS_HEADER_BYTES + SA_NOALLOC_MARK_BYTES];

namespace {
std::mutex g_noalloc_mu;
void* g_noalloc_addr[64] = {nullptr};

// Device address of g_noalloc_scratch on the current device, looked up once
// per device (host code cannot use the symbol itself as a device pointer).
sa_status noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail("sa_block_union_prefill_noalloc: cudaGetDevice", e);
  if (dev < 0 || dev >= 64) return fail(SA_ERR_UNSUPPORTED, "sa_block_union_prefill_noalloc: device %d >= 64", dev);
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (g_noalloc_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail("sa_block_union_prefill_noalloc: cudaGetSymbolAddress", e);
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return SA_OK;
}
}  // namespace

extern "C" sa_status sa_block_union_prefill_noalloc(const int32_t* idx, const int32_t* q_pos, const void* Q,
                                                    const void* K, const void* V, int S, int Nq, int Hq, int Hkv,
                                                    int d, int k, int block, float scale, int32_t* kv_indptr,
                                                    int32_t* kv_indices, void* O, sa_dtype out_dtype, void* stream) {
  const char* who = "sa_block_union_prefill_noalloc";
  if (S < 1 || Nq < 1 || Hq < 1 || Hkv < 1 || k < 1) return fail(SA_ERR_INVALID_ARG, "%s: sizes must be >= 1", who);
  if (d != 128) return fail(SA_ERR_UNSUPPORTED, "%s: d=%d (only 128 is built)", who, d);
  if (block != 64) return fail(SA_ERR_UNSUPPORTED, "%s: block=%d (only 64 is built)", who, block);
  const int64_t nb = ((int64_t)S + block - 1) / block;
  if (nb > SA_NOALLOC_MARK_BYTES)
    return fail(SA_ERR_UNSUPPORTED, "%s: S=%d needs %lld KV blocks; the static scratch holds at most %d (S <= %d)",
                who, S, (long long)nb, SA_NOALLOC_MARK_BYTES, SA_NOALLOC_MARK_BYTES * 64);
  if (Hq % Hkv != 0) return fail(SA_ERR_INVALID_ARG, "%s: Hq not a multiple of Hkv", who);
  if ((int64_t)Nq * (Hq / Hkv) > (1 << 30)) return fail(SA_ERR_INVALID_ARG, "%s: too many query rows", who);
  if (out_dtype != SA_BF16 && out_dtype != SA_F32) return fail(SA_ERR_INVALID_ARG, "%s: bad out_dtype", who);
  if (!idx || !q_pos || !Q || !K || !V || !kv_indptr || !kv_indices || !O)
    return fail(SA_ERR_INVALID_ARG, "%s: NULL pointer", who);
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(O, 16))
    return fail(SA_ERR_INVALID_ARG, "%s: Q, K, V, O must be 16-byte aligned", who);
  if (!(scale > 0.f)) return fail(SA_ERR_INVALID_ARG, "%s: scale must be > 0", who);
  void* scratch = nullptr;
  sa_status st = noalloc_scratch(&scratch);
  if (st != SA_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  // the previous call's status and marks are still in the array: start clean
  cudaError_t e = cudaMemsetAsync(scratch, 0, SA_WS_HEADER_BYTES, s);
  if (e != cudaSuccess) return cuda_fail("sa_block_union_prefill_noalloc clear", e);
  uint8_t* mark = reinterpret_cast<uint8_t*>(scratch) + SA_WS_HEADER_BYTES;
  e = sa::launch_block_union(idx, Nq, k, S, block, Hkv, mark, kv_indptr, kv_indices, status_of(scratch), s);
  if (e != cudaSuccess) return cuda_fail("sa_block_union_prefill_noalloc union", e);
  return prefill_attn(Q, K, V, q_pos, kv_indptr, kv_indices, S, Nq, Hq, Hkv, block, scale, O, out_dtype,
                      status_of(scratch), nullptr, 0, 0.f, nullptr, s, "sa_block_union_prefill_noalloc attention");
}
