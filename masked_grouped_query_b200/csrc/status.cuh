// status.cuh -- the library's sticky device-side status word.
//
// Kernels never trap.  When a bounded wait gives up (a barrier that did not
// complete within kWaitLimitNs) the kernel ORs a code into g_gqa_status,
// leaves its loops, releases what it holds and returns; the host reads the
// word with gqa_attn_status() after synchronising.
#pragma once

#include <stdint.h>

namespace gqa {

// Status bits (also listed in include/gqa_attn.h).
enum : uint32_t {
  kStatusTimeoutProducer = 1u << 0,   // loader waited too long for a free stage
  kStatusTimeoutConsumer = 1u << 1,   // compute warps waited too long for data
  kStatusTimeoutMma = 1u << 2,        // MMA issuer waited too long
  kStatusTimeoutSoftmax = 1u << 3,    // softmax warps waited too long
  kStatusTimeoutEpilogue = 1u << 4,   // epilogue waited too long
  kStatusTimeoutTest = 1u << 5,       // the bounded-wait self test expired
};

// Two seconds: far above any legitimate wait in these kernels.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// Defined here: the library is compiled as a single translation unit.
__device__ uint32_t g_gqa_status = 0;

__device__ __forceinline__ void report_status(uint32_t code) { atomicOr(&g_gqa_status, code); }

}  // namespace gqa
