// kda_prefill_api.cu -- C ABI of the chunked KDA prefill (include/kda_prefill.h):
// argument validation, the workspace size, and the three kernel launches of
// kda_prefill_kernel.cuh on the caller's stream.  Nothing here allocates or
// synchronises.
#include <atomic>
#include <cstdint>

#include "kda_decode.h"
#include "kda_host_util.h"
#include "kda_prefill.h"
#include "kda_prefill_kernel.cuh"

namespace {

using namespace kda_host;
namespace kp = kdap;

// Chunks of a run of T tokens; false on overflow of the workspace arithmetic.
bool workspace_floats(int64_t N, int64_t T, int64_t HV, int64_t* nchunks, int64_t* floats) {
  *nchunks = (T + kp::kC - 1) / kp::kC;
  int64_t units;
  return mul_ok(N, HV, &units) && mul_ok(units, *nchunks, floats) && mul_ok(*floats, kp::Workspace::kFloats, floats) &&
         !__builtin_add_overflow(*floats, kp::Workspace::kHeaderFloats, floats);
}

// Once per device: the three kernels' dynamic shared memory allowances.
cudaError_t prepare_kernels() {
  static std::atomic<uint64_t> ready{0};  // bit d: done on device d (d < 64)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  const uint64_t bit = dev < 64 ? (uint64_t{1} << dev) : 0;
  if (bit && (ready.load(std::memory_order_relaxed) & bit)) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(kp::kda_prefill_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kp::kChunkSmem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kp::kda_prefill_state_kernel<8, 256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kp::kStateSmem<8, 256>);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kp::kda_prefill_state_kernel<16, 256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kp::kStateSmem<16, 256>);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kp::kda_prefill_state_kernel<32, 256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kp::kStateSmem<32, 256>);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kp::kda_prefill_state_kernel<64, 512>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kp::kStateSmem<64, 512>);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kp::kda_prefill_output_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kp::kOutSmem);
  if (e == cudaSuccess && bit) ready.fetch_or(bit, std::memory_order_relaxed);
  return e;
}

// The current device's SM count, once per device.
int sm_count() {
  static std::atomic<int> cache[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  int v = dev < kMaxDevices ? cache[dev].load(std::memory_order_relaxed) : 0;
  if (v == 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    if (dev < kMaxDevices) cache[dev].store(v, std::memory_order_relaxed);
  }
  return v;
}

// Validation and the launches of the stages in [first, last] (0: chunk
// preparation, 1: state recurrence, 2: chunk outputs), in order.
kda_status prefill_stages(const void* q, const void* k, const void* v, const float* g, const float* beta,
                          float* state_pool, const int32_t* slot_idx, void* out, void* workspace,
                          int64_t workspace_bytes, int64_t N, int64_t T, int64_t HV, int64_t K, int64_t V,
                          float scale, kda_stream_t stream, int first, int last);

}  // namespace

extern "C" {

int64_t kda_prefill_workspace_bytes(int64_t N, int64_t T, int64_t HV, int64_t K, int64_t V) {
  if (N < 0 || T < 0 || HV < 0) return -1;
  if (K != kp::kK || V != kp::kV) return -1;
  if (N == 0 || T == 0 || HV == 0) return 0;
  int64_t nchunks, floats, bytes;
  if (!workspace_floats(N, T, HV, &nchunks, &floats) || !mul_ok(floats, 4, &bytes)) return -1;
  return bytes;
}

kda_status kda_prefill(const void* q, const void* k, const void* v, const float* g, const float* beta,
                       float* state_pool, const int32_t* slot_idx, void* out, void* workspace,
                       int64_t workspace_bytes, int64_t N, int64_t T, int64_t HV, int64_t K, int64_t V,
                       float scale, kda_stream_t stream) {
  return prefill_stages(q, k, v, g, beta, state_pool, slot_idx, out, workspace, workspace_bytes, N, T, HV, K, V,
                        scale, stream, 0, 2);
}

kda_status kda_prefill_stage(int32_t stage, const void* q, const void* k, const void* v, const float* g,
                             const float* beta, float* state_pool, const int32_t* slot_idx, void* out,
                             void* workspace, int64_t workspace_bytes, int64_t N, int64_t T, int64_t HV, int64_t K,
                             int64_t V, float scale, kda_stream_t stream) {
  if (stage < 0 || stage > 2) return KDA_ERR_INVALID_ARG;
  return prefill_stages(q, k, v, g, beta, state_pool, slot_idx, out, workspace, workspace_bytes, N, T, HV, K, V,
                        scale, stream, stage, stage);
}

}  // extern "C"

namespace {

kda_status prefill_stages(const void* q, const void* k, const void* v, const float* g, const float* beta,
                          float* state_pool, const int32_t* slot_idx, void* out, void* workspace,
                          int64_t workspace_bytes, int64_t N, int64_t T, int64_t HV, int64_t K, int64_t V,
                          float scale, kda_stream_t stream, int first, int last) {
  if (N < 0 || T < 0 || HV < 0 || K < 0 || V < 0 || workspace_bytes < 0) return KDA_ERR_INVALID_ARG;
  if (HV < 1 || K != kp::kK || V != kp::kV) return KDA_ERR_UNSUPPORTED;
  if (N == 0 || T == 0) return KDA_OK;  // nothing to do; no pointer is touched

  int64_t nchunks, floats, rows, hk, hv_v, out_elems, grid_chunks, grid_state;
  if (!workspace_floats(N, T, HV, &nchunks, &floats) || !mul_ok(N, T, &rows) || !mul_ok(HV, K, &hk) ||
      !mul_ok(HV, V, &hv_v) || !mul_ok(rows, hv_v, &out_elems) || out_elems > INT64_MAX / 8 ||
      !mul_ok(N * HV, nchunks, &grid_chunks) || grid_chunks > 0x7fffffffLL ||
      !mul_ok(N * HV, kp::kV / 8, &grid_state) || grid_state > 0x7fffffffLL || floats > INT64_MAX / 4 ||
      nchunks > 0x7fffffffLL)
    return KDA_ERR_UNSUPPORTED;

  if (!q || !k || !v || !g || !beta || !state_pool || !slot_idx || !out || !workspace) return KDA_ERR_INVALID_ARG;
  if (workspace_bytes < floats * 4) return KDA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(g, 16) || !aligned(state_pool, 16) ||
      !aligned(out, 16) || !aligned(workspace, 16) || !aligned(beta, 4) || !aligned(slot_idx, 4))
    return KDA_ERR_MISALIGNED;

  // out and the workspace are written: neither may overlap an input, the
  // pool's visible extent (slot 0 and its base address) or the other.
  const Range r_out = range_of(out, out_elems * 2);
  const Range r_ws = range_of(workspace, floats * 4);
  const Range inputs[] = {range_of(q, rows * hk * 2), range_of(k, rows * hk * 2), range_of(v, rows * hv_v * 2),
                          range_of(g, rows * hk * 4), range_of(beta, rows * HV * 4), range_of(slot_idx, N * 4)};
  const Range r_slot0 = range_of(state_pool, hk * V * 4);
  const uintptr_t pool_base = reinterpret_cast<uintptr_t>(state_pool);
  auto touches_pool = [&](Range r) { return overlaps(r, r_slot0) || (r.lo <= pool_base && pool_base < r.hi); };
  if (touches_pool(r_out) || touches_pool(r_ws) || overlaps(r_out, r_ws)) return KDA_ERR_ALIAS;
  for (const Range& r : inputs)
    if (overlaps(r, r_out) || overlaps(r, r_ws) || touches_pool(r)) return KDA_ERR_ALIAS;

  const kda_status dev = check_device();
  if (dev != KDA_OK) return dev;
  if (prepare_kernels() != cudaSuccess) return KDA_ERR_CUDA;

  kp::Params p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.g = g;
  p.beta = beta;
  p.state = state_pool;
  p.slot_idx = slot_idx;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.ws = static_cast<float*>(workspace);
  p.T = T;
  p.HV = HV;
  p.nchunks = static_cast<int32_t>(nchunks);
  p.scale = scale;

  cudaLaunchConfig_t cfg = {};
  cfg.stream = reinterpret_cast<cudaStream_t>(stream);
  auto run = [&](auto kernel, int64_t grid, int threads, int smem) {
    cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.blockDim = dim3(static_cast<unsigned>(threads), 1, 1);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    return cudaLaunchKernelEx(&cfg, kernel, p);
  };
  const int bv = kp::state_tile_width(N * HV, sm_count());
  const int64_t grid_tiles = N * HV * (kp::kV / bv);
  if (first <= 0 && 0 <= last &&
      run(kp::kda_prefill_chunk_kernel, grid_chunks, kp::kChunkThreads, kp::kChunkSmem) != cudaSuccess)
    return KDA_ERR_CUDA;
  if (first <= 1 && 1 <= last) {
    cudaError_t e_state;
    if (bv == 8) e_state = run(kp::kda_prefill_state_kernel<8, 256>, grid_tiles, 256, kp::kStateSmem<8, 256>);
    else if (bv == 16) e_state = run(kp::kda_prefill_state_kernel<16, 256>, grid_tiles, 256, kp::kStateSmem<16, 256>);
    else if (bv == 32) e_state = run(kp::kda_prefill_state_kernel<32, 256>, grid_tiles, 256, kp::kStateSmem<32, 256>);
    else e_state = run(kp::kda_prefill_state_kernel<64, 512>, grid_tiles, 512, kp::kStateSmem<64, 512>);
    if (e_state != cudaSuccess) return KDA_ERR_CUDA;
  }
  if (first <= 2 && 2 <= last &&
      run(kp::kda_prefill_output_kernel, grid_chunks, kp::kOutThreads, kp::kOutSmem) != cudaSuccess)
    return KDA_ERR_CUDA;
  return KDA_OK;
}

}  // namespace

// ---------------------------------------------------------------- kda_prefill_no_alloc
// Scratch for callers that cannot allocate (see include/kda_prefill.h): a
// file-scope device array, 256-byte aligned like a cudaMalloc block.  In host
// code its name stands for the variable, not for a device address: the
// address comes from cudaGetSymbolAddress, once per device, below.
static __device__ __align__(256) unsigned char g_prefill_scratch[KDA_PREFILL_NO_ALLOC_SCRATCH_BYTES];

namespace {

std::atomic<void*> g_scratch_addr[kMaxDevices];  // per device, found on its first call

// The scratch array's address on the current device (nullptr if the lookup fails).
void* scratch_on_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return nullptr;
  if (dev < kMaxDevices) {
    void* known = g_scratch_addr[dev].load(std::memory_order_acquire);
    if (known != nullptr) return known;
  }
  void* addr = nullptr;
  if (cudaGetSymbolAddress(&addr, g_prefill_scratch) != cudaSuccess) return nullptr;
  if (dev < kMaxDevices) g_scratch_addr[dev].store(addr, std::memory_order_release);
  return addr;
}

}  // namespace

extern "C" kda_status kda_prefill_no_alloc(const void* q, const void* k, const void* v, const float* g,
                                           const float* beta, float* state_pool, const int32_t* slot_idx,
                                           void* out, int64_t N, int64_t T, int64_t HV, int64_t K, int64_t V,
                                           float scale, kda_stream_t stream) {
  const int64_t need = kda_prefill_workspace_bytes(N, T, HV, K, V);
  if (need < 0) {  // the sizes kda_prefill would refuse: let it give the reason
    return kda_prefill(q, k, v, g, beta, state_pool, slot_idx, out, nullptr, 0, N, T, HV, K, V, scale, stream);
  }
  if (need > KDA_PREFILL_NO_ALLOC_SCRATCH_BYTES) return KDA_ERR_SCRATCH_LIMIT;
  if (N == 0 || T == 0 || HV == 0)  // nothing to do; no pointer (and no scratch) is touched
    return kda_prefill(q, k, v, g, beta, state_pool, slot_idx, out, nullptr, 0, N, T, HV, K, V, scale, stream);
  const kda_status dev = check_device();
  if (dev != KDA_OK) return dev;
  void* const scratch = scratch_on_current_device();
  if (scratch == nullptr) return KDA_ERR_CUDA;
  return kda_prefill(q, k, v, g, beta, state_pool, slot_idx, out, scratch, KDA_PREFILL_NO_ALLOC_SCRATCH_BYTES, N, T,
                     HV, K, V, scale, stream);
}
