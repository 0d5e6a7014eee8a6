// Device-side timeline of the decode step (a tracing build only).
//
// Built with -DSA_TIMELINE (cross_layer_shared_b200/timeline.py does this, into
// a separate library), every SA_TL(kernel, slot) point writes the %globaltimer
// value of the CTA's thread that reaches it into
//   timeline[(kernel * kTimelineCtas + blockIdx.x) * kTimelineSlots + slot]
// when the buffer has been set with that translation unit's setter
// (sa_timeline_set_<unit>).  Without SA_TIMELINE the points compile to
// nothing and no setter exists: the library proper carries no tracing.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace sa {
constexpr int kTimelineCtas = 4096;
constexpr int kTimelineSlots = 64;
enum : int { kTlIndexer = 0, kTlTopk = 1, kTlAttn = 2, kTlAttnSmall = 3 };
}  // namespace sa

#ifdef SA_TIMELINE
static __device__ unsigned long long* g_sa_timeline;
#define SA_TL(kid, slot)                                                                          \
  do {                                                                                            \
    if (g_sa_timeline != nullptr) {                                                               \
      unsigned long long t_;                                                                      \
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                                      \
      g_sa_timeline[((size_t)(kid) * sa::kTimelineCtas + blockIdx.x) * sa::kTimelineSlots + (slot)] = t_; \
    }                                                                                             \
  } while (0)
#define SA_TL_SETTER(name) \
  extern "C" int name(void* p) { return (int)cudaMemcpyToSymbol(g_sa_timeline, &p, sizeof p); }
#else
#define SA_TL(kid, slot) \
  do {                   \
  } while (0)
#define SA_TL_SETTER(name)
#endif
