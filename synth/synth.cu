// CUDA twin of the counter-based generator in synth/__init__.py.
//
// Fills large bf16 tensors on the device with the same bits the host
// generator produces for the same (seed, stream id, flat index): element i
// is the i-th SplitMix64 output of the stream key (Steele, Lea, Flood,
// OOPSLA 2014, finaliser "Mix13"), turned into an Irwin-Hall n=4 sample by
// integer adds and one fp32 multiply by sqrt(3)/65536, then scaled and
// rounded to bf16 (nearest-even).  It holds none of the attention method's
// arithmetic; both the oracle side and the CUDA side of a parity check take
// their inputs from this generator and its host twin.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

__host__ __device__ inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ inline uint16_t normal_bf16(uint64_t key, uint64_t i, float scale) {
  const uint64_t h = mix64(key + (i + 1ull) * kGamma);
  const uint32_t s = (uint32_t)(h & 0xFFFFu) + (uint32_t)((h >> 16) & 0xFFFFu) +
                     (uint32_t)((h >> 32) & 0xFFFFu) + (uint32_t)(h >> 48);
  const float ih_scale = __uint_as_float(0x37DDB3D7u);  // sqrt(3)/65536 in fp32
  float x = __fmul_rn((float)((int32_t)s - 131070), ih_scale);
  x = __fmul_rn(x, scale);
  return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

__global__ void fill_normal_bf16_kernel(uint16_t* __restrict__ out, int64_t n, uint64_t key,
                                        int64_t offset, float scale) {
  const int64_t n8 = n / 8;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < n8; v += stride) {
    const uint64_t i0 = (uint64_t)(offset + v * 8);
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t lo = normal_bf16(key, i0 + 2 * j, scale);
      const uint32_t hi = normal_bf16(key, i0 + 2 * j + 1, scale);
      w[j] = lo | (hi << 16);
    }
    reinterpret_cast<uint4*>(out)[v] = make_uint4(w[0], w[1], w[2], w[3]);
  }
  for (int64_t i = n8 * 8 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
    out[i] = normal_bf16(key, (uint64_t)(offset + i), scale);
}

}  // namespace

extern "C" {

// stream key of (seed, tid): mix64(seed * GAMMA + tid)
uint64_t synth_stream_key(uint64_t seed, uint64_t tid) { return mix64(seed * kGamma + tid); }

// out[i] = bf16(scale * N01(seed, tid, offset + i)), i in [0, n).  `out` must be
// 16-byte aligned.  Returns the cudaError_t of the launch.
int synth_fill_normal_bf16(void* out, int64_t n, uint64_t seed, uint64_t tid, int64_t offset,
                           float scale, cudaStream_t stream) {
  if (n <= 0) return 0;
  if (((uintptr_t)out & 15u) != 0) return (int)cudaErrorInvalidValue;
  const uint64_t key = synth_stream_key(seed, tid);
  int blocks = (int)((n / 8 + 255) / 256);
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (blocks < 1) blocks = 1;
  fill_normal_bf16_kernel<<<blocks, 256, 0, stream>>>(reinterpret_cast<uint16_t*>(out), n, key,
                                                      offset, scale);
  return (int)cudaGetLastError();
}

}  // extern "C"
