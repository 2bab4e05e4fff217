// kda_decode_api.cu -- C ABI of the recurrent KDA decode library (see
// include/kda_decode.h for the operation, layouts, ownership and errors).
//
// Host side only: argument validation, a per-device compute-capability cache
// (queried once per device, as the FlashInfer #4562 review of `CheckTarget`
// asks for a latency-sensitive decode path), and one kernel launch on the
// caller's stream.  Nothing here allocates, synchronises or falls back to
// another implementation.
#include <atomic>
#include <cstddef>
#include <cstdint>

#include "kda_decode.h"
#include "kda_decode_kernel.cuh"

namespace {

constexpr int kMaxDevices = 64;
std::atomic<int32_t> g_cc_cache[kMaxDevices];  // 0 = unknown, else major*10 + minor

kda_status check_device() {
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

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct Range {
  uintptr_t lo, hi;  // [lo, hi)
};
Range range_of(const void* p, int64_t bytes) {
  const uintptr_t lo = reinterpret_cast<uintptr_t>(p);
  return Range{lo, lo + static_cast<uintptr_t>(bytes)};
}
bool overlaps(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi; }

// Multiply non-negative sizes, flagging overflow of int64.
bool mul_ok(int64_t a, int64_t b, int64_t* r) { return !__builtin_mul_overflow(a, b, r); }

kda_status launch(const void* q, const void* k, const void* v, const float* g, const float* beta,
                  void* state_pool, const int32_t* slot_idx, const void* gate,
                  const void* norm_weight, float eps, void* out, int64_t N, int64_t T, int64_t HV,
                  int64_t K, int64_t V, float scale, kda_stream_t stream, bool gated, bool bf16_state) {
  // ---- sizes
  if (N < 0 || T < 0 || HV < 0 || K < 0 || V < 0) return KDA_ERR_INVALID_ARG;
  if (gated && !(eps >= 0.0f && eps <= 3.0e38f)) return KDA_ERR_INVALID_ARG;  // also rejects NaN
  if (HV < 1) return KDA_ERR_UNSUPPORTED;
  if (K != 64 && K != 128 && K != 256) return KDA_ERR_UNSUPPORTED;
  if (V < kda::kBV || V % kda::kBV != 0) return KDA_ERR_UNSUPPORTED;
  const int64_t tiles = V / kda::kBV;
  if (gated && tiles > kda::kMaxClusterTiles) return KDA_ERR_UNSUPPORTED;
  if (N == 0 || T == 0) return KDA_OK;  // nothing to do; no pointer is touched

  int64_t rows, qk_elems, v_elems, grid;
  if (!mul_ok(N, T, &rows) || !mul_ok(rows, HV, &rows) || !mul_ok(rows, K, &qk_elems) ||
      !mul_ok(rows, V, &v_elems) || qk_elems > (INT64_MAX / 4) || v_elems > (INT64_MAX / 4))
    return KDA_ERR_UNSUPPORTED;
  if (!mul_ok(N, HV, &grid) || !mul_ok(grid, tiles, &grid) || grid > 0x7fffffffLL)
    return KDA_ERR_UNSUPPORTED;

  // ---- pointers
  if (!q || !k || !v || !g || !beta || !state_pool || !slot_idx || !out) return KDA_ERR_INVALID_ARG;
  if (gated && (!gate || !norm_weight)) return KDA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(g, 16) ||
      !aligned(state_pool, 16) || !aligned(out, 16) || !aligned(beta, 4) || !aligned(slot_idx, 4))
    return KDA_ERR_MISALIGNED;
  if (gated && (!aligned(gate, 16) || !aligned(norm_weight, 16))) return KDA_ERR_MISALIGNED;

  // ---- aliasing: out must not overlap any input or the pool
  const Range r_out = range_of(out, v_elems * 2);
  const Range inputs[] = {
      range_of(q, qk_elems * 2), range_of(k, qk_elems * 2), range_of(v, v_elems * 2),
      range_of(g, qk_elems * 4), range_of(beta, rows * 4), range_of(slot_idx, N * 4),
      range_of(gated ? gate : nullptr, gated ? v_elems * 2 : 0),
      range_of(gated ? norm_weight : nullptr, gated ? V * 2 : 0)};
  // The pool's extent depends on slot values held on the device; the visible
  // part is slot 0 plus the base address itself.
  const Range r_slot0 = range_of(state_pool, HV * K * V * (bf16_state ? 2 : 4));
  const uintptr_t pool_base = reinterpret_cast<uintptr_t>(state_pool);
  auto touches_pool = [&](Range r) {
    return overlaps(r, r_slot0) || (r.lo <= pool_base && pool_base < r.hi);
  };
  if (touches_pool(r_out)) return KDA_ERR_ALIAS;
  for (const Range& r : inputs) {
    if (r.hi == r.lo) continue;
    if (overlaps(r, r_out) || touches_pool(r)) return KDA_ERR_ALIAS;
  }

  // ---- device
  const kda_status dev = check_device();
  if (dev != KDA_OK) return dev;

  kda::Params p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.g = g;
  p.beta = beta;
  p.state = state_pool;
  p.slot_idx = slot_idx;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.gate = static_cast<const __nv_bfloat16*>(gate);
  p.norm_weight = static_cast<const __nv_bfloat16*>(norm_weight);
  p.T = T;
  p.HV = HV;
  p.V = V;
  p.tiles = static_cast<int32_t>(tiles);
  p.scale = scale;
  p.eps = eps;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kda::kThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = reinterpret_cast<cudaStream_t>(stream);
  // Programmatic stream serialization: the kernel waits for earlier work in
  // the stream (griddepcontrol.wait) before its first global access, so the
  // launch itself may overlap the tail of the previous kernel.
  cudaLaunchAttribute attr[2];
  cfg.attrs = attr;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.numAttrs = 1;
  if (gated) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = static_cast<unsigned>(tiles);
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
  }

  cudaError_t err = cudaErrorInvalidValue;
  const bool multi = T > 1;
  const bool v128 = V == 128;
  // One instantiation per (K, V fixed at 128 or not, gated, state type); T == 1
  // and T > 1 (chunked) kernels.
#define KDA_LAUNCH(KERNEL, KK, VV, GG)                                                      \
  do {                                                                                      \
    if (bf16_state) err = cudaLaunchKernelEx(&cfg, kda::KERNEL<KK, VV, GG, __nv_bfloat16>, p); \
    else err = cudaLaunchKernelEx(&cfg, kda::KERNEL<KK, VV, GG, float>, p);                  \
  } while (0)
#define KDA_LAUNCH_V(KK, GG)                                                 \
  do {                                                                       \
    if (multi) {                                                             \
      if (v128) KDA_LAUNCH(kda_decode_chunked_kernel, KK, 128, GG);          \
      else KDA_LAUNCH(kda_decode_chunked_kernel, KK, 0, GG);                 \
    } else {                                                                 \
      if (v128) KDA_LAUNCH(kda_decode_kernel, KK, 128, GG);                  \
      else KDA_LAUNCH(kda_decode_kernel, KK, 0, GG);                         \
    }                                                                        \
  } while (0)
#define KDA_LAUNCH_K(KK)                   \
  do {                                     \
    if (gated) KDA_LAUNCH_V(KK, true);     \
    else KDA_LAUNCH_V(KK, false);          \
  } while (0)
  switch (K) {
    case 64: KDA_LAUNCH_K(64); break;
    case 128: KDA_LAUNCH_K(128); break;
    case 256: KDA_LAUNCH_K(256); break;
    default: return KDA_ERR_UNSUPPORTED;
  }
#undef KDA_LAUNCH_K
#undef KDA_LAUNCH_V
#undef KDA_LAUNCH
  return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

}  // namespace

extern "C" {

kda_status kda_decode(const void* q, const void* k, const void* v, const float* g, const float* beta,
                      float* state_pool, const int32_t* slot_idx, void* out, int64_t N, int64_t T,
                      int64_t HV, int64_t K, int64_t V, float scale, kda_stream_t stream) {
  return launch(q, k, v, g, beta, state_pool, slot_idx, nullptr, nullptr, 0.0f, out, N, T, HV, K, V,
                scale, stream, /*gated=*/false, /*bf16_state=*/false);
}

kda_status kda_decode_gated_rmsnorm(const void* q, const void* k, const void* v, const float* g,
                                    const float* beta, float* state_pool, const int32_t* slot_idx,
                                    const void* gate, const void* norm_weight, float eps, void* out,
                                    int64_t N, int64_t T, int64_t HV, int64_t K, int64_t V,
                                    float scale, kda_stream_t stream) {
  return launch(q, k, v, g, beta, state_pool, slot_idx, gate, norm_weight, eps, out, N, T, HV, K, V,
                scale, stream, /*gated=*/true, /*bf16_state=*/false);
}

kda_status kda_decode_bf16_state(const void* q, const void* k, const void* v, const float* g,
                                 const float* beta, void* state_pool, const int32_t* slot_idx, void* out,
                                 int64_t N, int64_t T, int64_t HV, int64_t K, int64_t V, float scale,
                                 kda_stream_t stream) {
  return launch(q, k, v, g, beta, state_pool, slot_idx, nullptr, nullptr, 0.0f, out, N, T, HV, K, V,
                scale, stream, /*gated=*/false, /*bf16_state=*/true);
}

kda_status kda_decode_gated_rmsnorm_bf16_state(const void* q, const void* k, const void* v,
                                               const float* g, const float* beta, void* state_pool,
                                               const int32_t* slot_idx, const void* gate,
                                               const void* norm_weight, float eps, void* out, int64_t N,
                                               int64_t T, int64_t HV, int64_t K, int64_t V, float scale,
                                               kda_stream_t stream) {
  return launch(q, k, v, g, beta, state_pool, slot_idx, gate, norm_weight, eps, out, N, T, HV, K, V,
                scale, stream, /*gated=*/true, /*bf16_state=*/true);
}

const char* kda_status_string(kda_status status) {
  switch (status) {
    case KDA_OK: return "ok";
    case KDA_ERR_INVALID_ARG: return "invalid argument (null pointer, negative size or bad eps)";
    case KDA_ERR_UNSUPPORTED: return "unsupported size (K must be 64/128/256, V a multiple of 32, "
                                     "V <= 256 when gated, HV >= 1)";
    case KDA_ERR_ALIAS: return "output overlaps an input or the state pool";
    case KDA_ERR_MISALIGNED: return "misaligned pointer (16 bytes for tensors, 4 for beta/slot_idx)";
    case KDA_ERR_DEVICE: return "current device is not compute capability 10.0 (sm_100a)";
    case KDA_ERR_CUDA: return "CUDA launch failed";
  }
  return "unknown status";
}

int32_t kda_abi_version(void) { return (1 << 16) | 1; }

}  // extern "C"
