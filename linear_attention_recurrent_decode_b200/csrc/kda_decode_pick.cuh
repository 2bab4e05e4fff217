// kda_decode_pick.cuh -- host-side choice of the decode kernel instantiation.
//
// pick_decode_kernel<K> maps a call's form (plain or gated, one token or a
// chunked run, V fixed at 128 or not, pool layout and element type, input
// form) to one instantiation of the kernels in kda_decode_kernel.cuh, makes
// its one-time launch settings and returns its address and dynamic shared
// memory.  Each K is instantiated in its own translation unit
// (kda_decode_k64.cu, kda_decode_k128.cu, kda_decode_k256.cu) so that the
// library's 288 kernels compile in parallel.
#pragma once

#include <atomic>
#include <cstdint>

#include "kda_decode_kernel.cuh"

namespace kda {

struct KernelChoice {
  bool gated;
  bool multi;         // T > 1: the chunked kernel
  bool v128;          // V == 128: compile-time row strides
  bool vk;            // [V][K] pool blocks
  bool bf16_state;
  int form;           // InputForm
  int tiles;          // V / kBV (the cluster size of the gated kernels)
  bool check_launch;  // also check, once per kernel and device, that the launch can run
};

// Once per kernel and device: check that the kernel loads on the device and,
// for a cluster launch of `cluster` CTAs, that at least one such cluster fits
// (kda_decode_host makes this check before it enqueues its copy in).
template <auto Kernel>
cudaError_t launchable(int cluster, int smem) {
  static std::atomic<uint64_t> ready{0};  // bit d: checked on device d (d < 64)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  const uint64_t bit = dev < 64 ? (uint64_t{1} << dev) : 0;
  if (bit && (ready.load(std::memory_order_relaxed) & bit)) return cudaSuccess;
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, Kernel);
  if (e == cudaSuccess && cluster > 1) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(cluster), 1, 1);
    cfg.blockDim = dim3(kda::kThreads, 1, 1);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = static_cast<unsigned>(cluster);
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&clusters, Kernel, &cfg);
    if (e == cudaSuccess && clusters < 1) e = cudaErrorInvalidConfiguration;
  }
  if (e == cudaSuccess && bit) ready.fetch_or(bit, std::memory_order_relaxed);
  return e;
}

// Once per kernel and device: let the kernel take `bytes` of dynamic shared
// memory (the [V][K] staging buffer; above 48 KB this needs the opt-in) and
// prefer the shared-memory carveout.
template <auto Kernel>
cudaError_t allow_dynamic_smem(int bytes) {
  static std::atomic<uint64_t> ready{0};  // bit d: done on device d (d < 64)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  const uint64_t bit = dev < 64 ? (uint64_t{1} << dev) : 0;
  if (bit && (ready.load(std::memory_order_relaxed) & bit)) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(Kernel, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess && bit) ready.fetch_or(bit, std::memory_order_relaxed);
  return e;
}


// The device error word of K's translation unit (g_device_error is static:
// one per unit, written only by that unit's kernels); clear resets it.
template <int K>
cudaError_t device_error_word(int32_t* word, bool clear) {
  cudaError_t e = cudaMemcpyFromSymbol(word, g_device_error, sizeof(int32_t));
  if (e == cudaSuccess && clear) {
    const int32_t zero = 0;
    e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof zero);
  }
  return e;
}

template <int K>
cudaError_t pick_decode_kernel(const KernelChoice& c, const void** func, int* smem_out) {
  cudaError_t err = cudaSuccess;
  const bool gated = c.gated, vk = c.vk, bf16_state = c.bf16_state;
  const int form = c.form;
  // One instantiation per (K, V fixed at 128 or not, gated, state type, input
  // form, state layout); T == 1 and T > 1 (chunked) kernels.
#define KDA_PICK_ONE(KERNEL, KK, VV, GG, STT, RR, VKK)                                               \
  do {                                                                                                \
    constexpr auto kern = KERNEL<KK, VV, GG, STT, RR, VKK>;                                           \
    constexpr int smem = KERNEL##_dyn_smem<KK, STT, RR, VKK>;                                         \
    *smem_out = smem;                                                                                 \
    err = smem ? allow_dynamic_smem<kern>(smem) : cudaSuccess;                                        \
    if (err == cudaSuccess && c.check_launch) err = launchable<kern>(gated ? c.tiles : 1, smem);      \
    *func = reinterpret_cast<const void*>(kern);                                                      \
  } while (0)
#define KDA_PICK_ST(KERNEL, KK, VV, GG, RR)                                                           \
  do {                                                                                                \
    if (vk) {                                                                                         \
      if (bf16_state) KDA_PICK_ONE(KERNEL, KK, VV, GG, __nv_bfloat16, RR, true);                      \
      else KDA_PICK_ONE(KERNEL, KK, VV, GG, float, RR, true);                                         \
    } else {                                                                                          \
      if (bf16_state) KDA_PICK_ONE(KERNEL, KK, VV, GG, __nv_bfloat16, RR, false);                     \
      else KDA_PICK_ONE(KERNEL, KK, VV, GG, float, RR, false);                                        \
    }                                                                                                 \
  } while (0)
#define KDA_PICK(KERNEL, KK, VV, GG)                                          \
  do {                                                                        \
    if (form == kInRaw) KDA_PICK_ST(KERNEL, KK, VV, GG, kInRaw);              \
    else if (form == kInDense) KDA_PICK_ST(KERNEL, KK, VV, GG, kInDense);     \
    else KDA_PICK_ST(KERNEL, KK, VV, GG, kInStrided);                         \
  } while (0)
#define KDA_PICK_V(KK, GG)                                              \
  do {                                                                  \
    if (form == kInGeneral) {                                           \
      if (c.multi) {                                                    \
        if (bf16_state) KDA_PICK_ONE(kda_decode_chunked_kernel, KK, 0, GG, __nv_bfloat16, kInGeneral, false); \
        else KDA_PICK_ONE(kda_decode_chunked_kernel, KK, 0, GG, float, kInGeneral, false);                     \
      } else {                                                          \
        if (bf16_state) KDA_PICK_ONE(kda_decode_kernel, KK, 0, GG, __nv_bfloat16, kInGeneral, false);         \
        else KDA_PICK_ONE(kda_decode_kernel, KK, 0, GG, float, kInGeneral, false);                             \
      }                                                                 \
    } else if (c.multi) {                                               \
      if (c.v128) KDA_PICK(kda_decode_chunked_kernel, KK, 128, GG);     \
      else KDA_PICK(kda_decode_chunked_kernel, KK, 0, GG);              \
    } else {                                                            \
      if (c.v128) KDA_PICK(kda_decode_kernel, KK, 128, GG);             \
      else KDA_PICK(kda_decode_kernel, KK, 0, GG);                      \
    }                                                                   \
  } while (0)
  if (gated) KDA_PICK_V(K, true);
  else KDA_PICK_V(K, false);
#undef KDA_PICK_V
#undef KDA_PICK
#undef KDA_PICK_ST
#undef KDA_PICK_ONE
  return err;
}

}  // namespace kda
