// Device status block kept at the start of every workspace.
//
//   word 0        status code (0 = ok), written once with atomicCAS
//   words 2..9    four int64 detail values of the first error
//                 (kernel id, element index, offending value, bound)
//
// Kernels never trap: an out-of-range input or a wait that gives up is
// recorded here and the element is skipped.
#pragma once

#include <stdint.h>

namespace sa {

enum : int {
  kOk = 0,
  kErrInvalidArg = 1,
  kErrUnsupported = 2,
  kErrWorkspace = 3,
  kErrCuda = 4,
  kErrTimeout = 5,
  kErrDevice = 6,
};

enum : int {
  kKernIndexer = 1,
  kKernTopk = 2,
  kKernAttn = 3,
  kKernCombine = 4,
  kKernUnion = 5,
  kKernIndexerPrefill = 6,
  kKernRoute = 7,
  kKernWaitProbe = 8,
  kKernCp = 9,
};

struct DeviceStatus {
  int code;
  int pad;
  long long detail[4];
};

constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s per wait

__device__ __forceinline__ void report(DeviceStatus* st, int code, long long kernel, long long a,
                                       long long b, long long c) {
  if (st == nullptr) return;
  if (atomicCAS(&st->code, 0, code) == 0) {
    st->detail[0] = kernel;
    st->detail[1] = a;
    st->detail[2] = b;
    st->detail[3] = c;
    __threadfence();
  }
}

}  // namespace sa
