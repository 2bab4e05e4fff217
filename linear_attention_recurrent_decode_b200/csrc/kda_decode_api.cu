// kda_decode_api.cu -- C ABI of the recurrent KDA decode library (see
// include/kda_decode.h for the operation, layouts, ownership and errors).
//
// Host side only: argument validation, a per-device compute-capability cache
// (queried once per device, as the FlashInfer #4562 review of `CheckTarget`
// asks for a latency-sensitive decode path), and one kernel launch on the
// caller's stream (kda_decode_host adds the copies in and out around it).
// Nothing here allocates or falls back to another implementation, and no
// step entry point synchronises (kda_decode_device_error, a diagnostic, reads
// the kernels' error word synchronously).
#include <atomic>
#include <cstddef>
#include <cstdint>

#include "kda_decode.h"
#include "kda_decode_pick.cuh"
#include "kda_host_util.h"

// The kernels are instantiated in kda_decode_k{64,128,256}.cu.
namespace kda {
extern template cudaError_t pick_decode_kernel<64>(const KernelChoice&, const void**, int*);
extern template cudaError_t pick_decode_kernel<128>(const KernelChoice&, const void**, int*);
extern template cudaError_t pick_decode_kernel<256>(const KernelChoice&, const void**, int*);
extern template cudaError_t device_error_word<64>(int32_t*, bool);
extern template cudaError_t device_error_word<128>(int32_t*, bool);
extern template cudaError_t device_error_word<256>(int32_t*, bool);
}  // namespace kda

namespace {

using namespace kda_host;


// Host staging of kda_decode_host: the step's inputs are copied from host_in to
// dev_in before the kernel, the output from out to host_out after it.  With a
// copy stream (kda_decode_host_pipelined) the copy in runs there, between a
// wait for `free_ev` and a record of `ready_ev`; the kernel waits for
// `ready_ev` and is followed by a record of `free_ev`.
struct HostCopies {
  const void* host_in;
  void* dev_in;
  int64_t in_bytes;
  void* host_out;
  cudaStream_t copy_stream = nullptr;
  cudaEvent_t ready_ev = nullptr;
  cudaEvent_t free_ev = nullptr;
};

kda_status launch(const kda_decode_args& a, bool gated, kda_stream_t stream, const HostCopies* hc = nullptr) {
  const int64_t N = a.N, T = a.T, HV = a.HV, K = a.K, V = a.V;
  if (hc && (hc->in_bytes < 0 || (hc->in_bytes > 0 && (!hc->host_in || !hc->dev_in)) || !hc->host_out))
    return KDA_ERR_INVALID_ARG;
  // ---- sizes
  if (N < 0 || T < 0 || HV < 0 || K < 0 || V < 0 || a.num_slots < 0) return KDA_ERR_INVALID_ARG;
  if (gated && !(a.eps >= 0.0f && a.eps <= 3.0e38f)) return KDA_ERR_INVALID_ARG;  // also rejects NaN
  if (a.state_dtype != KDA_STATE_FP32 && a.state_dtype != KDA_STATE_BF16) return KDA_ERR_INVALID_ARG;
  if (a.state_layout != KDA_LAYOUT_KV && a.state_layout != KDA_LAYOUT_VK) return KDA_ERR_INVALID_ARG;
  if (HV < 1 || K < 1 || K > 256 || V < 1) return KDA_ERR_UNSUPPORTED;
  // The vectorised kernels take K in {64, 128, 256} and V a multiple of 32;
  // any other K <= 256 and V run the general (masked, element-wise) form of
  // the same kernels on K padded to 64, 128 or 256 rows.
  const bool general = !((K == 64 || K == 128 || K == 256) && V % kda::kBV == 0);
  const int64_t K_pad = K <= 64 ? 64 : (K <= 128 ? 128 : 256);
  const int64_t tiles = (V + kda::kBV - 1) / kda::kBV;
  if (gated && tiles > kda::kMaxClusterTiles) return KDA_ERR_UNSUPPORTED;
  if (general && (a.state_layout != KDA_LAYOUT_KV || a.raw_gate != nullptr || a.raw_beta != nullptr))
    return KDA_ERR_UNSUPPORTED;  // the general form takes [K][V] blocks and activated g, beta
  if (N == 0 || T == 0) return KDA_OK;  // nothing to do; no pointer is touched

  int64_t rows, hk, hvv, grid, out_elems;
  if (!mul_ok(N, T, &rows) || !mul_ok(HV, K, &hk) || !mul_ok(HV, V, &hvv) ||
      !mul_ok(rows, hvv, &out_elems) || out_elems > (INT64_MAX / 4))
    return KDA_ERR_UNSUPPORTED;
  if (!mul_ok(N, HV, &grid) || !mul_ok(grid, tiles, &grid) || grid > 0x7fffffffLL)
    return KDA_ERR_UNSUPPORTED;

  // ---- which decay and beta inputs: (g, beta) or the raw serving form
  const bool raw = a.raw_gate != nullptr || a.raw_beta != nullptr;
  if (raw) {
    if (!a.raw_gate || !a.raw_beta || !a.A_log || !a.dt_bias || a.g || a.beta) return KDA_ERR_INVALID_ARG;
  } else if (!a.g || !a.beta) {
    return KDA_ERR_INVALID_ARG;
  }

  // ---- pointers
  if (!a.q || !a.k || !a.v || !a.state_pool || !a.slot_idx || !a.out) return KDA_ERR_INVALID_ARG;
  if (gated && (!a.gate || !a.norm_weight)) return KDA_ERR_INVALID_ARG;
  const void* gsrc = raw ? a.raw_gate : static_cast<const void*>(a.g);
  const void* bsrc = raw ? a.raw_beta : static_cast<const void*>(a.beta);
  const bool bf16_pool = a.state_dtype == KDA_STATE_BF16;
  // The vectorised kernels read 16-byte pieces; the general form reads element
  // by element and needs only each element's own alignment.
  const uintptr_t va = general ? 2 : 16, ga = general ? 4 : 16, sa = general ? (bf16_pool ? 2 : 4) : 16;
  if (!aligned(a.q, va) || !aligned(a.k, va) || !aligned(a.v, va) || !aligned(gsrc, ga) ||
      !aligned(a.state_pool, sa) || !aligned(a.out, va) || !aligned(bsrc, raw ? 2 : 4) ||
      !aligned(a.slot_idx, 4))
    return KDA_ERR_MISALIGNED;
  if (raw && (!aligned(a.dt_bias, 16) || !aligned(a.A_log, 4))) return KDA_ERR_MISALIGNED;
  if (a.status && !aligned(a.status, 4)) return KDA_ERR_MISALIGNED;
  if (gated && (!aligned(a.gate, va) || !aligned(a.norm_weight, va))) return KDA_ERR_MISALIGNED;

  // ---- row strides: at least one row, and (vectorised kernels) 16-byte aligned rows
  const int64_t g_elem = raw ? 2 : 4;
  if (a.q_row_stride < hk || a.k_row_stride < hk || a.v_row_stride < hvv || a.g_row_stride < hk ||
      a.beta_row_stride < HV || (gated && a.gate_row_stride < hvv))
    return KDA_ERR_INVALID_ARG;
  if (!general && (a.q_row_stride % 8 || a.k_row_stride % 8 || a.v_row_stride % 8 ||
                   (a.g_row_stride * g_elem) % 16 || (gated && a.gate_row_stride % 8)))
    return KDA_ERR_MISALIGNED;

  // ---- aliasing: out must not overlap any input or the pool
  int64_t bq, bk, bv, bg, bb, bz = 0;
  if (!span_bytes(rows, a.q_row_stride, hk, 2, &bq) || !span_bytes(rows, a.k_row_stride, hk, 2, &bk) ||
      !span_bytes(rows, a.v_row_stride, hvv, 2, &bv) ||
      !span_bytes(rows, a.g_row_stride, hk, g_elem, &bg) ||
      !span_bytes(rows, a.beta_row_stride, HV, raw ? 2 : 4, &bb) ||
      (gated && !span_bytes(rows, a.gate_row_stride, hvv, 2, &bz)))
    return KDA_ERR_UNSUPPORTED;
  const Range r_out = range_of(a.out, out_elems * 2);
  const Range inputs[] = {
      range_of(a.q, bq), range_of(a.k, bk), range_of(a.v, bv), range_of(gsrc, bg), range_of(bsrc, bb),
      range_of(a.slot_idx, N * 4), range_of(gated ? a.gate : nullptr, gated ? bz : 0),
      range_of(gated ? a.norm_weight : nullptr, gated ? V * 2 : 0),
      range_of(raw ? a.A_log : nullptr, raw ? HV * 4 : 0),
      range_of(raw ? a.dt_bias : nullptr, raw ? hk * 4 : 0)};
  // The pool's extent: all num_slots blocks when the call declares the pool's
  // size; otherwise it depends on slot values held on the device, and the
  // visible part is slot 0 plus the base address itself.
  const bool bf16_state = a.state_dtype == KDA_STATE_BF16;
  int64_t block_bytes, pool_bytes = 0;
  if (!mul_ok(hk, V * (bf16_state ? 2 : 4), &block_bytes) ||
      (a.num_slots > 0 && !mul_ok(block_bytes, a.num_slots, &pool_bytes)))
    return KDA_ERR_UNSUPPORTED;
  const Range r_pool = range_of(a.state_pool, a.num_slots > 0 ? pool_bytes : block_bytes);
  const uintptr_t pool_base = reinterpret_cast<uintptr_t>(a.state_pool);
  auto touches_pool = [&](Range r) {
    return overlaps(r, r_pool) || (r.lo <= pool_base && pool_base < r.hi);
  };
  if (touches_pool(r_out)) return KDA_ERR_ALIAS;
  if (hc && hc->in_bytes > 0 && touches_pool(range_of(hc->dev_in, hc->in_bytes))) return KDA_ERR_ALIAS;
  const Range r_status = range_of(a.status, a.status ? 4 : 0);
  if (a.status && (overlaps(r_status, r_out) || touches_pool(r_status))) return KDA_ERR_ALIAS;
  for (const Range& r : inputs) {
    if (r.hi == r.lo) continue;
    if (overlaps(r, r_out) || touches_pool(r) || (a.status && overlaps(r, r_status))) return KDA_ERR_ALIAS;
  }

  // ---- device
  const kda_status dev = check_device();
  if (dev != KDA_OK) return dev;

  kda::ParamsEx p;
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.k = static_cast<const __nv_bfloat16*>(a.k);
  p.v = static_cast<const __nv_bfloat16*>(a.v);
  p.g = a.g;
  p.beta = a.beta;
  p.state = a.state_pool;
  p.slot_idx = a.slot_idx;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.gate = static_cast<const __nv_bfloat16*>(a.gate);
  p.norm_weight = static_cast<const __nv_bfloat16*>(a.norm_weight);
  p.raw_gate = static_cast<const __nv_bfloat16*>(a.raw_gate);
  p.A_log = a.A_log;
  p.dt_bias = a.dt_bias;
  p.raw_beta = static_cast<const __nv_bfloat16*>(a.raw_beta);
  p.q_rs = a.q_row_stride;
  p.k_rs = a.k_row_stride;
  p.v_rs = a.v_row_stride;
  p.g_rs = a.g_row_stride;
  p.b_rs = a.beta_row_stride;
  p.z_rs = gated ? a.gate_row_stride : 0;
  p.T = T;
  p.HV = HV;
  p.V = V;
  p.tiles = static_cast<int32_t>(tiles);
  p.scale = a.scale;
  p.eps = a.eps;
  p.num_slots = a.num_slots;
  p.status = a.status;
  p.k_rt = static_cast<int32_t>(K);

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

  // Input form: raw serving inputs; dense rows (offsets from the shape alone,
  // whatever entry point was called) when the slots are unchecked; any other
  // row strides, or checked slots (only the larger parameter block carries the
  // pool size and the status word).
  const bool dense = a.q_row_stride == hk && a.k_row_stride == hk && a.v_row_stride == hvv &&
                     a.g_row_stride == hk && a.beta_row_stride == HV && (!gated || a.gate_row_stride == hvv) &&
                     a.num_slots == 0;
  const int form = general ? kda::kInGeneral : raw ? kda::kInRaw : dense ? kda::kInDense : kda::kInStrided;

  // Pick the kernel (and make its dynamic shared memory allowance) before
  // anything is enqueued.
  const bool vk = a.state_layout == KDA_LAYOUT_VK;
  const void* func = nullptr;
  int smem = 0;
  kda::KernelChoice choice;
  choice.gated = gated;
  choice.multi = T > 1;
  choice.v128 = V == 128;
  choice.vk = vk;
  choice.bf16_state = bf16_state;
  choice.form = form;
  choice.tiles = static_cast<int>(tiles);
  choice.check_launch = hc != nullptr;
  cudaError_t err = cudaErrorInvalidValue;
  switch (K_pad) {
    case 64: err = kda::pick_decode_kernel<64>(choice, &func, &smem); break;
    case 128: err = kda::pick_decode_kernel<128>(choice, &func, &smem); break;
    case 256: err = kda::pick_decode_kernel<256>(choice, &func, &smem); break;
    default: return KDA_ERR_UNSUPPORTED;
  }
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  if (err != cudaSuccess || func == nullptr) return KDA_ERR_CUDA;
  if (hc) {
    // With host copies around the step, the launch was checked above (once per
    // kernel and device: the kernel loads, a cluster fits) before the copy in
    // is enqueued.
    if (hc->copy_stream) {
      if (cudaStreamWaitEvent(hc->copy_stream, hc->free_ev, 0) != cudaSuccess) return KDA_ERR_CUDA;
      if (hc->in_bytes > 0 &&
          cudaMemcpyAsync(hc->dev_in, hc->host_in, static_cast<size_t>(hc->in_bytes), cudaMemcpyHostToDevice,
                          hc->copy_stream) != cudaSuccess)
        return KDA_ERR_CUDA;
      if (cudaEventRecord(hc->ready_ev, hc->copy_stream) != cudaSuccess ||
          cudaStreamWaitEvent(cfg.stream, hc->ready_ev, 0) != cudaSuccess)
        return KDA_ERR_CUDA;
    } else if (hc->in_bytes > 0 &&
               cudaMemcpyAsync(hc->dev_in, hc->host_in, static_cast<size_t>(hc->in_bytes), cudaMemcpyHostToDevice,
                               cfg.stream) != cudaSuccess) {
      return KDA_ERR_CUDA;
    }
  }
  // The dense form's kernels take the smaller parameter block, which is the
  // leading part of p.
  void* kargs[] = {&p};
  err = cudaLaunchKernelExC(&cfg, func, kargs);
  if (err != cudaSuccess) return KDA_ERR_CUDA;
  if (hc && hc->copy_stream && cudaEventRecord(hc->free_ev, cfg.stream) != cudaSuccess) return KDA_ERR_CUDA;
  if (hc && cudaMemcpyAsync(hc->host_out, a.out, static_cast<size_t>(out_elems) * 2, cudaMemcpyDeviceToHost,
                            cfg.stream) != cudaSuccess)
    return KDA_ERR_CUDA;
  return KDA_OK;
}

// Dense (contiguous) arguments of the four fixed-layout entry points.
kda_decode_args dense_args(const void* q, const void* k, const void* v, const float* g, const float* beta,
                           void* state_pool, int32_t state_dtype, const int32_t* slot_idx, const void* gate,
                           const void* norm_weight, float eps, void* out, int64_t N, int64_t T, int64_t HV,
                           int64_t K, int64_t V, float scale) {
  kda_decode_args a = {};
  a.q = q;
  a.q_row_stride = HV * K;
  a.k = k;
  a.k_row_stride = HV * K;
  a.v = v;
  a.v_row_stride = HV * V;
  a.g = g;
  a.g_row_stride = HV * K;
  a.beta = beta;
  a.beta_row_stride = HV;
  a.state_pool = state_pool;
  a.state_dtype = state_dtype;
  a.state_layout = KDA_LAYOUT_KV;
  a.slot_idx = slot_idx;
  a.gate = gate;
  a.gate_row_stride = HV * V;
  a.norm_weight = norm_weight;
  a.eps = eps;
  a.out = out;
  a.N = N;
  a.T = T;
  a.HV = HV;
  a.K = K;
  a.V = V;
  a.scale = scale;
  return a;
}

}  // namespace

extern "C" {

kda_status kda_decode(const void* q, const void* k, const void* v, const float* g, const float* beta,
                      float* state_pool, const int32_t* slot_idx, void* out, int64_t N, int64_t T,
                      int64_t HV, int64_t K, int64_t V, float scale, kda_stream_t stream) {
  return launch(dense_args(q, k, v, g, beta, state_pool, KDA_STATE_FP32, slot_idx, nullptr, nullptr, 0.0f,
                           out, N, T, HV, K, V, scale),
                /*gated=*/false, stream);
}

kda_status kda_decode_gated_rmsnorm(const void* q, const void* k, const void* v, const float* g,
                                    const float* beta, float* state_pool, const int32_t* slot_idx,
                                    const void* gate, const void* norm_weight, float eps, void* out,
                                    int64_t N, int64_t T, int64_t HV, int64_t K, int64_t V,
                                    float scale, kda_stream_t stream) {
  return launch(dense_args(q, k, v, g, beta, state_pool, KDA_STATE_FP32, slot_idx, gate, norm_weight, eps,
                           out, N, T, HV, K, V, scale),
                /*gated=*/true, stream);
}

kda_status kda_decode_bf16_state(const void* q, const void* k, const void* v, const float* g,
                                 const float* beta, void* state_pool, const int32_t* slot_idx, void* out,
                                 int64_t N, int64_t T, int64_t HV, int64_t K, int64_t V, float scale,
                                 kda_stream_t stream) {
  return launch(dense_args(q, k, v, g, beta, state_pool, KDA_STATE_BF16, slot_idx, nullptr, nullptr, 0.0f,
                           out, N, T, HV, K, V, scale),
                /*gated=*/false, stream);
}

kda_status kda_decode_gated_rmsnorm_bf16_state(const void* q, const void* k, const void* v,
                                               const float* g, const float* beta, void* state_pool,
                                               const int32_t* slot_idx, const void* gate,
                                               const void* norm_weight, float eps, void* out, int64_t N,
                                               int64_t T, int64_t HV, int64_t K, int64_t V, float scale,
                                               kda_stream_t stream) {
  return launch(dense_args(q, k, v, g, beta, state_pool, KDA_STATE_BF16, slot_idx, gate, norm_weight, eps,
                           out, N, T, HV, K, V, scale),
                /*gated=*/true, stream);
}

kda_status kda_decode_ex(const kda_decode_args* args, kda_stream_t stream) {
  if (args == nullptr) return KDA_ERR_INVALID_ARG;
  if ((args->gate == nullptr) != (args->norm_weight == nullptr)) return KDA_ERR_INVALID_ARG;
  return launch(*args, /*gated=*/args->gate != nullptr, stream);
}

kda_status kda_decode_host(const kda_decode_args* args, const void* host_in, void* dev_in, int64_t in_bytes,
                           void* host_out, kda_stream_t stream) {
  if (args == nullptr) return KDA_ERR_INVALID_ARG;
  if ((args->gate == nullptr) != (args->norm_weight == nullptr)) return KDA_ERR_INVALID_ARG;
  const HostCopies hc{host_in, dev_in, in_bytes, host_out};
  return launch(*args, /*gated=*/args->gate != nullptr, stream, &hc);
}

kda_status kda_decode_host_pipelined(const kda_decode_args* args, const void* host_in, void* dev_in,
                                     int64_t in_bytes, void* host_out, kda_stream_t stream,
                                     kda_stream_t copy_stream, kda_event_t staging_ready,
                                     kda_event_t staging_free) {
  if (args == nullptr || stream == nullptr || copy_stream == nullptr || stream == copy_stream ||
      staging_ready == nullptr || staging_free == nullptr)
    return KDA_ERR_INVALID_ARG;
  if ((args->gate == nullptr) != (args->norm_weight == nullptr)) return KDA_ERR_INVALID_ARG;
  HostCopies hc{host_in, dev_in, in_bytes, host_out};
  hc.copy_stream = reinterpret_cast<cudaStream_t>(copy_stream);
  hc.ready_ev = reinterpret_cast<cudaEvent_t>(staging_ready);
  hc.free_ev = reinterpret_cast<cudaEvent_t>(staging_free);
  return launch(*args, /*gated=*/args->gate != nullptr, stream, &hc);
}

int32_t kda_host_memory_is_mapped(const void* p, int64_t bytes) {
  if (p == nullptr || bytes <= 0) return 0;
  const unsigned char* last = static_cast<const unsigned char*>(p) + (bytes - 1);
  for (const void* q : {p, static_cast<const void*>(last)}) {
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, q) != cudaSuccess) {
      cudaGetLastError();  // an unregistered pointer is an answer here, not a sticky error
      return 0;
    }
    if (attr.type != cudaMemoryTypeHost || attr.devicePointer != q || attr.hostPointer != q) return 0;
  }
  // both ends in one allocation: the device addresses of the two ends differ
  // by exactly the host distance (checked above: they equal the host addresses)
  return 1;
}

const char* kda_status_string(kda_status status) {
  switch (status) {
    case KDA_OK: return "ok";
    case KDA_ERR_INVALID_ARG:
      return "invalid argument (null pointer, negative size, bad eps, short row stride or mixed input forms)";
    case KDA_ERR_UNSUPPORTED: return "unsupported size or form (K in 1..256, V >= 1, V <= 256 when gated, "
                                     "HV >= 1; K outside {64,128,256} or V not a multiple of 32 only with "
                                     "[K][V] blocks and activated g, beta; prefill: K = V = 128)";
    case KDA_ERR_ALIAS: return "output overlaps an input or the state pool";
    case KDA_ERR_MISALIGNED: return "misaligned pointer or row stride";
    case KDA_ERR_DEVICE: return "current device is not compute capability 10.0 (sm_100a)";
    case KDA_ERR_CUDA: return "CUDA launch failed";
    case KDA_ERR_SCRATCH_LIMIT:
      return "sizes need more scratch than kda_prefill_no_alloc's fixed array holds (use kda_prefill)";
  }
  return "unknown status";
}

kda_status kda_decode_device_error(int32_t* word, int32_t clear) {
  if (!word) return KDA_ERR_INVALID_ARG;
  int32_t w64 = 0, w128 = 0, w256 = 0;
  if (kda::device_error_word<64>(&w64, clear != 0) != cudaSuccess ||
      kda::device_error_word<128>(&w128, clear != 0) != cudaSuccess ||
      kda::device_error_word<256>(&w256, clear != 0) != cudaSuccess)
    return KDA_ERR_CUDA;
  *word = w64 | w128 | w256;
  return KDA_OK;
}

int32_t kda_abi_version(void) { return (1 << 16) | 9; }

}  // extern "C"
