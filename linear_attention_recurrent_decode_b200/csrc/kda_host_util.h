// kda_host_util.h -- host-side helpers shared by the library's entry points:
// the per-device compute-capability check and the pointer-range arithmetic of
// the argument validation.  Host code only.
#pragma once

#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "kda_decode.h"

namespace kda_host {

constexpr int kMaxDevices = 64;
inline std::atomic<int32_t> g_cc_cache[kMaxDevices];  // 0 = unknown, else major*10 + minor

inline kda_status check_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return KDA_ERR_DEVICE;
  int32_t cc = dev < kMaxDevices ? g_cc_cache[dev].load(std::memory_order_relaxed) : 0;
  if (cc == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return KDA_ERR_DEVICE;
    cc = major * 10 + minor;
    if (dev < kMaxDevices) g_cc_cache[dev].store(cc, std::memory_order_relaxed);
  }
  // The library carries sm_100a code only; it runs on compute capability 10.0.
  return cc == 100 ? KDA_OK : KDA_ERR_DEVICE;
}

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct Range {
  uintptr_t lo, hi;  // [lo, hi)
};
inline Range range_of(const void* p, int64_t bytes) {
  const uintptr_t lo = reinterpret_cast<uintptr_t>(p);
  return Range{lo, lo + static_cast<uintptr_t>(bytes)};
}
inline bool overlaps(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi; }

// Multiply non-negative sizes, flagging overflow of int64.
inline bool mul_ok(int64_t a, int64_t b, int64_t* r) { return !__builtin_mul_overflow(a, b, r); }

// Bytes spanned by `rows` rows of `width` elements, `stride` elements apart.
inline bool span_bytes(int64_t rows, int64_t stride, int64_t width, int64_t elem, int64_t* bytes) {
  int64_t a;
  if (!mul_ok(rows - 1, stride, &a) || __builtin_add_overflow(a, width, &a)) return false;
  return mul_ok(a, elem, bytes);
}

}  // namespace kda_host
