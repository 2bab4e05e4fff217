// kda_decode_kernel.cuh -- sm_100a kernels of the recurrent KDA decode step.
//
// One CTA of 128 threads owns one (sequence n, value head h, 32-column value
// tile) of the fp32 state S[K][V] (V contiguous).  The CTA
//   1. reads slot_idx[n] and issues every 128-bit load of its K x 32 state tile
//      at once (8..32 KiB in flight per CTA), straight into registers: the tile
//      is touched exactly once, so staging it in shared memory would only add
//      a copy (a bulk-TMA staging of the same tile measured no faster on B200).
//      A pool with [V][K] blocks (K contiguous) is the exception: its tile
//      moves through shared memory so that global accesses stay whole-line
//      (TileIO below);
//   2. for each token: decays its rows by exp(g), forms the two reductions
//      S'^T k and S'^T q over K (in-thread over its rows, a reduce-scatter of
//      warp shuffles across the 4 row groups of a warp, shared memory across
//      the 4 warps), the correction u = beta (v - S'^T k), the rank-1 write
//      S += k u^T and the readout o = scale (S'^T q + (q.k) u), which equals
//      scale S^T q of the updated state without a second pass over it;
//   3. writes the tile back to the same slot once, after the last token.
// The state therefore crosses HBM exactly once in each direction per call.
//
// All per-element arithmetic uses Blackwell's packed fp32x2 instructions
// (__fmul2_rn / __ffma2_rn / __fadd2_rn: two IEEE round-to-nearest lanes per
// instruction).  The kernel is a single wave at serving batch sizes, so every
// CTA computes at the same moment after its loads land: instruction count is
// on the critical path, and the packed forms halve it.
//
// Multi-token calls (T > 1) use a second kernel that takes the tokens in
// chunks of up to four.  Within a chunk every token's reductions run against
// the chunk-start state, with the cumulative decays folded into per-row
// coefficients, and the tokens are coupled through small per-head scalars:
// with d_t = exp(g_t), A_t = d_0 ... d_t and B(s->t) = d_{s+1} ... d_t,
//   R_t = S0^T (A_t k_t),   Q_t = S0^T (A_t q_t),
//   M[t][s] = sum_i k_s,i B(s->t)_i k_t,i  (s < t),
//   P[t][s] = sum_i k_s,i B(s->t)_i q_t,i  (s <= t),
//   u_t = beta_t (v_t - R_t - sum_{s<t} M[t][s] u_s),
//   o_t = scale (Q_t + sum_{s<=t} P[t][s] u_s),
//   S_end = A_last S0 + sum_t (B(t->last) k_t) u_t^T,
// which is the token-by-token recurrence regrouped (equal in exact
// arithmetic): one cross-thread exchange per chunk instead of one per token,
// and each state element is read and written once per chunk.
//
// The gated variant launches the V/32 tiles of one (n, h) as a thread-block
// cluster.  One token: every tile hands its outputs and their sum of squares
// to the tile-0 CTA through distributed shared memory and an mbarrier, and
// that CTA alone applies the RMS over V, the norm weight and the sigmoid gate
// before the bf16 store.  Several tokens: each CTA pushes its per-token sums of
// o^2 into every peer and one cluster barrier per chunk completes the RMS.
//
// Inputs may be row-strided views (q, k, v as slices of one packed buffer),
// and the serving form takes a raw bf16 gate and beta activated in the kernel
// (input form kInRaw): g = -exp(A_log[h]) softplus(raw_gate + dt_bias[h]),
// beta = sigmoid(raw_beta).  The sources name these inputs but print no
// activation; this is the usual KDA gate and is documented as a reading.
//
// The state pool is fp32 or bf16 (template parameter ST).  A bf16 pool is
// widened exactly on load, all arithmetic is fp32, and the state is rounded
// to nearest even once, when it is written back at the end of the call.
//
// Launch overlap: kernels are launched with programmatic stream
// serialization.  Every global access of a CTA comes after griddepcontrol.wait
// (all work earlier in the stream complete and visible), and a CTA lets the
// next kernel in the stream start launching once it is about to write its
// state back, so the next call's launch overlaps this call's stores.  The
// state is written with streaming (evict-first) stores: it is not read again
// before the next decode step.
//
// No tensor cores: the step is a chain of mat-vec products with O(1) flops
// per state byte, far below any tensor-core ridge point; the roofline is HBM.
//
// Sources (pages by title): vLLM #57585 "Tune recurrent KDA launch
// configuration on SM90" (BF16 inputs, FP32 recurrent state, K = V = 128;
// Triton grid over (N*HV, V tiles)); FlashInfer #4562 "feat(cake_kda): add
// optimized H12 packed decode across SM100 family" (value tiles per head,
// 128-thread CTAs, cp.async staging; state_indices and scale as launch
// arguments); b12x #249 "feat(gdn): add direct single-token KDA decode"
// (decode then gated RMS norm of the output).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>

namespace kda {

constexpr int kThreads = 128;               // 4 warps
constexpr int kWarps = kThreads / 32;
constexpr int kBV = 32;                     // value columns per CTA
constexpr int kColQuads = kBV / 4;          // float4 column groups per row segment (8)
constexpr int kRowGroups = 32 / kColQuads;  // row groups per warp (4)
constexpr int kMaxClusterTiles = 8;         // portable cluster size bound
constexpr int kChunk = 4;                   // tokens per chunk in the multi-token kernel

struct Params {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const float* g;
  const float* beta;
  void* state;  // fp32 or bf16 [num_slots, HV, K, V] (the kernel's ST)
  const int32_t* slot_idx;
  __nv_bfloat16* out;
  const __nv_bfloat16* gate;         // gated variant only
  const __nv_bfloat16* norm_weight;  // gated variant only
  int64_t T;
  int64_t HV;
  int64_t V;
  int32_t tiles;  // V / kBV
  float scale;
  float eps;
};

// Row-strided views and the serving input form.  Only the kernels of those
// forms take this larger block: the dense kernels keep the small one (a larger
// parameter block alone measurably slowed them, through register allocation).
struct ParamsEx : Params {
  // Serving input form: g = -exp(A_log[h]) softplus(raw_gate + dt_bias[h]),
  // beta = sigmoid(raw_beta).
  const __nv_bfloat16* raw_gate;
  const float* A_log;    // [HV]
  const float* dt_bias;  // [HV, K]
  const __nv_bfloat16* raw_beta;
  // Row strides, in elements, between consecutive (n, t) rows of each input;
  // element (n, t, h, i) of q sits at (n*T + t)*q_rs + h*K + i (v and gate with
  // V, beta with 1).  g_rs / b_rs apply to g / beta or to raw_gate / raw_beta.
  int64_t q_rs, k_rs, v_rs, g_rs, b_rs, z_rs;
  // Checked slots: num_slots > 0 makes a row whose slot is >= num_slots an
  // inactive row and stores 1 to *status (when not null).
  int64_t num_slots;
  int32_t* status;
  // General form only: the run-time key width (the kernel's K is its padded
  // row count).
  int32_t k_rt;
};

// How a kernel addresses its per-token inputs and which decay/beta inputs it
// reads.  Dense inputs take their row offsets from the shape alone, so the
// offsets of q, k, v, g, beta and out share one (n, t, h) row index.
enum InputForm : int {
  kInDense = 0,    // q, k, v, g, beta, gate dense [N, T, HV, ...]; activated g and beta
  kInStrided = 1,  // row-strided views; activated g and beta
  kInRaw = 2,      // row-strided views; raw gate and beta, activated in the kernel
  // Any K <= the kernel's K and any V: row-strided views read element by
  // element, key rows >= k_rt and value columns >= V masked to zero (never
  // read or written).  [K][V] pool blocks, activated g and beta.
  kInGeneral = 3,
};
template <int IN>
using ParamsOf = typename std::conditional<IN == kInDense, Params, ParamsEx>::type;

// Whether row n takes part in the call: slot >= 0, and (checked forms with a
// declared pool size) slot < num_slots.  The first thread of a CTA that meets
// an out-of-range slot raises the status word.  Every CTA of one (n, h) sees
// the same slot, so the decision is uniform over a cluster.
template <int IN, typename P>
__device__ __forceinline__ bool row_active(const P& p, int32_t slot) {
  if constexpr (IN != kInDense) {
    if (p.num_slots > 0 && slot >= p.num_slots) {
      if (threadIdx.x == 0 && p.status != nullptr) atomicOr(p.status, 1);
      return false;
    }
  }
  return slot >= 0;
}

// Which input an offset is taken in (selects the row stride).
enum InputRow : int { kRowQ, kRowK, kRowG, kRowV, kRowZ, kRowB };

// Element offset of head h in (n, t) row nt of input WHICH, `width` elements
// per head.  `row` = nt * HV + h is the dense row index, computed once by the
// caller (recomputing it per input measurably slowed the one-token kernel).
template <int IN, int WHICH, typename P>
__device__ __forceinline__ int64_t in_off(const P& p, int64_t row, int64_t nt, int64_t h, int64_t width) {
  if constexpr (IN == kInDense) {
    return row * width;
  } else {
    const int64_t rs = WHICH == kRowQ   ? p.q_rs
                       : WHICH == kRowK ? p.k_rs
                       : WHICH == kRowG ? p.g_rs
                       : WHICH == kRowV ? p.v_rs
                       : WHICH == kRowZ ? p.z_rs
                                        : p.b_rs;
    return nt * rs + h * width;
  }
}

// ---------------------------------------------------------------- helpers
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ float bf16_at(const uint32_t* w, int i) {
  return (i & 1) ? bf16hi(w[i >> 1]) : bf16lo(w[i >> 1]);
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&p);
}
__device__ __forceinline__ float2 f2(float a) { return make_float2(a, a); }

// Four consecutive state values of one key row, in the pool's element type
// ST: fp32 (128-bit accesses) or bf16 (64-bit accesses; widened exactly on
// load, rounded to nearest even on store).  Stores stream (evict-first): the
// state is not read again before the next decode step.
template <typename ST>
struct StateIO;
template <>
struct StateIO<float> {
  static __device__ __forceinline__ void load(float2 (&s)[2], const float* p) {
    const float4 x = *reinterpret_cast<const float4*>(p);
    s[0] = make_float2(x.x, x.y);
    s[1] = make_float2(x.z, x.w);
  }
  static __device__ __forceinline__ void store(float* p, const float2 (&s)[2]) {
    __stcs(reinterpret_cast<float4*>(p), make_float4(s[0].x, s[0].y, s[1].x, s[1].y));
  }
};
template <>
struct StateIO<__nv_bfloat16> {
  static __device__ __forceinline__ void load(float2 (&s)[2], const __nv_bfloat16* p) {
    const uint2 x = *reinterpret_cast<const uint2*>(p);
    s[0] = make_float2(bf16lo(x.x), bf16hi(x.x));
    s[1] = make_float2(bf16lo(x.y), bf16hi(x.y));
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, const float2 (&s)[2]) {
    __stcs(reinterpret_cast<uint2*>(p), make_uint2(pack_bf16x2(s[0].x, s[0].y), pack_bf16x2(s[1].x, s[1].y)));
  }
};

// RPT consecutive bf16 values (RPT = 4: 8 bytes; RPT % 8 == 0: 16-byte chunks).
template <int RPT>
__device__ __forceinline__ void ld_bf16_rows(uint32_t (&w)[RPT / 2], const __nv_bfloat16* p) {
  if constexpr (RPT % 8 == 0) {
#pragma unroll
    for (int i = 0; i < RPT / 8; ++i) {
      const uint4 x = __ldg(reinterpret_cast<const uint4*>(p) + i);
      w[4 * i + 0] = x.x; w[4 * i + 1] = x.y; w[4 * i + 2] = x.z; w[4 * i + 3] = x.w;
    }
  } else {
    static_assert(RPT == 4, "rows per thread: 4 or a multiple of 8");
    const uint2 x = __ldg(reinterpret_cast<const uint2*>(p));
    w[0] = x.x; w[1] = x.y;
  }
}
template <int NF>
__device__ __forceinline__ void ld_f32_rows(float (&d)[NF], const float* p) {
#pragma unroll
  for (int i = 0; i < NF / 4; ++i) {
    const float4 x = __ldg(reinterpret_cast<const float4*>(p) + i);
    d[4 * i + 0] = x.x; d[4 * i + 1] = x.y; d[4 * i + 2] = x.z; d[4 * i + 3] = x.w;
  }
}

// General form: RPT consecutive rows starting at key row r0, element by element,
// zero for rows at or past k_rt.
template <int RPT>
__device__ __forceinline__ void ld_bf16_rows_masked(uint32_t (&w)[RPT / 2], const __nv_bfloat16* p, int r0,
                                                    int k_rt) {
  const unsigned short* u = reinterpret_cast<const unsigned short*>(p);
#pragma unroll
  for (int i = 0; i < RPT / 2; ++i) {
    const uint32_t lo = r0 + 2 * i < k_rt ? __ldg(u + 2 * i) : 0u;
    const uint32_t hi = r0 + 2 * i + 1 < k_rt ? __ldg(u + 2 * i + 1) : 0u;
    w[i] = lo | (hi << 16);
  }
}
template <int NF>
__device__ __forceinline__ void ld_f32_rows_masked(float (&d)[NF], const float* p, int r0, int k_rt) {
#pragma unroll
  for (int i = 0; i < NF; ++i) d[i] = r0 + i < k_rt ? __ldg(p + i) : 0.f;
}
// Four consecutive bf16 values of a row, element by element, zero at or past
// column `lim` (the row's value count) from column `c`.
__device__ __forceinline__ void ld_bf16x4_masked(uint32_t (&w)[2], const __nv_bfloat16* p, int64_t c, int64_t lim) {
  const unsigned short* u = reinterpret_cast<const unsigned short*>(p);
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const uint32_t lo = c + 2 * i < lim ? __ldg(u + 2 * i) : 0u;
    const uint32_t hi = c + 2 * i + 1 < lim ? __ldg(u + 2 * i + 1) : 0u;
    w[i] = lo | (hi << 16);
  }
}
__device__ __forceinline__ void st_bf16x4_masked(__nv_bfloat16* p, const float (&y)[4], int64_t c, int64_t lim) {
#pragma unroll
  for (int j = 0; j < 4; ++j)
    if (c + j < lim) p[j] = __float2bfloat16_rn(y[j]);
}

// General form: a thread's state tile (rows r0 .. r0+RPT-1, columns c .. c+3)
// element by element in a [K][V] block of run-time size, masked to the block.
template <typename ST, int RPT>
struct MaskedTile {
  static __device__ __forceinline__ ST* base(void* pool, int64_t slot, int64_t HV, int64_t h, int64_t k_rt,
                                             int64_t V, int r0, int64_t c) {
    return static_cast<ST*>(pool) + (slot * HV + h) * k_rt * V + static_cast<int64_t>(r0) * V + c;
  }
  static __device__ __forceinline__ float rd(const float* p) { return *p; }
  static __device__ __forceinline__ float rd(const __nv_bfloat16* p) { return __bfloat162float(*p); }
  static __device__ __forceinline__ void wr(float* p, float x) { __stcs(p, x); }
  static __device__ __forceinline__ void wr(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }
  static __device__ __forceinline__ void load(float2 (&s)[RPT][2], const ST* b, int64_t V, int r0, int k_rt,
                                              int64_t c) {
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
      const bool row = r0 + i < k_rt;
      float x[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) x[j] = (row && c + j < V) ? rd(b + i * V + j) : 0.f;
      s[i][0] = make_float2(x[0], x[1]);
      s[i][1] = make_float2(x[2], x[3]);
    }
  }
  static __device__ __forceinline__ void store(ST* b, const float2 (&s)[RPT][2], int64_t V, int r0, int k_rt,
                                               int64_t c) {
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
      if (r0 + i >= k_rt) continue;
      const float x[4] = {s[i][0].x, s[i][0].y, s[i][1].x, s[i][1].y};
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (c + j < V) wr(b + i * V + j, x[j]);
    }
  }
};

// Inputs of one token for one thread: its RPT key rows of q, k, g, its 4 value
// columns of v (and of the gate z), and beta.
template <int RPT>
struct TokenIn {
  uint32_t q[RPT / 2], k[RPT / 2];
  float g[RPT];
  uint32_t v[2];
  float beta;
};

// ---------------------------------------------------------------- serving-form activations
// softplus(x) = log(1 + e^x), exact to fp32 rounding for every x (for x > 15
// the correction log1p(e^-x) is below half an ulp of x).
__device__ __forceinline__ float softplus_f(float x) { return x > 15.f ? x : log1pf(expf(x)); }
__device__ __forceinline__ float sigmoid_f(float x) { return 1.0f / (1.0f + expf(-x)); }

// ---------------------------------------------------------------- cp.async
__device__ __forceinline__ uint32_t smem_u32(const void* ptr) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(ptr));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* mbar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(mbar)), "r"(count) : "memory");
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// Wait for phase `parity` of the mbarrier with cluster-scope acquire (it also
// sees what other CTAs of the cluster wrote before their release-arrives on
// it), giving up after `limit` polls (false then): no kernel waits without
// bound.
__device__ __forceinline__ bool mbar_wait_cluster_bounded(uint64_t* mbar, uint32_t parity, uint32_t limit) {
  for (uint32_t i = 0; i < limit; ++i) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(done)
        : "r"(smem_u32(mbar)), "r"(parity)
        : "memory");
    if (done) return true;
  }
  return false;
}
// Polls before a wait gives up: each try_wait suspends for a hardware-chosen
// interval, so this is seconds, against microseconds for what is awaited.
constexpr uint32_t kWaitPolls = 1u << 24;

// Device-side error word of the kernels of one translation unit (one per key
// size K): a kernel that gave up a bounded wait stores kDeviceErrorTimeout
// here (read and cleared by the host through kda_decode_device_error).
static __device__ int32_t g_device_error;
constexpr int32_t kDeviceErrorTimeout = 1;

// ---------------------------------------------------------------- cluster
__device__ __forceinline__ uint32_t cluster_map(uint32_t local_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local_addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_store_f32(uint32_t cluster_addr, float x) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(cluster_addr), "f"(x) : "memory");
}
__device__ __forceinline__ void cluster_store_f32x4(uint32_t cluster_addr, float a, float b, float c, float d) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(cluster_addr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}
// Arrive on an mbarrier in another CTA of the cluster, releasing this
// thread's earlier writes (to that CTA's shared memory included) at cluster scope.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// ---------------------------------------------------------------- programmatic dependent launch
__device__ __forceinline__ void wait_prior_grids() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void allow_next_grid() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- state tile I/O
// A thread's state tile: key rows r0 .. r0+RPT-1 of the value columns
// c .. c+3 (c = col0 + 4 cq), held as s[row][pair] (pair 0: columns c, c+1;
// pair 1: c+2, c+3).
//   VK = false, pool blocks [K][V]: row i of the thread's tile is four
//     consecutive values at base + i * V, base = element (r0, c); a warp's
//     16-byte accesses cover 4 rows x 128 bytes.
//   VK = true, pool blocks [V][K] (key index fastest, FlashInfer #4562's
//     layout): the CTA's 32 value columns are 32 runs of K contiguous values.
//     Read straight into the thread layout above, a warp access would touch 8
//     runs at half a line each (measured 1.6x slower), so the tile moves
//     through shared memory: cp.async copies the whole tile in 16-byte pieces
//     (a warp copies whole runs), then each thread reads its rows from the
//     staged columns; the write-back goes the same way in reverse.  Piece p of
//     staged column c sits at piece p ^ ((c >> 2) & 7), so the eight column
//     quads that a quarter-warp reads at once fall in eight different banks.
template <typename ST, bool VK, int K, int RPT>
struct TileIO {
  static constexpr int kE = 16 / static_cast<int>(sizeof(ST));  // elements per 16-byte piece
  static_assert(K / kE >= 8, "the swizzle permutes pieces within groups of eight");
  // Staging buffer of the [V][K] form, in dynamic shared memory (the launch
  // gives it kStageBytes; the [K][V] form takes none).
  struct Stage {
    alignas(16) ST v[VK ? kBV * K : 1];
  };
  static constexpr int kStageBytes = VK ? static_cast<int>(sizeof(Stage)) : 0;
  // Staged position of element (column c, key row r).
  static __device__ __forceinline__ int at(int c, int r) {
    return c * K + (((r / kE) ^ ((c >> 2) & 7)) * kE) + r % kE;
  }

  // KV: the thread's first element; VK: the first element of the CTA's tile.
  static __device__ __forceinline__ ST* base(void* pool, int64_t slot, int64_t HV, int64_t h, int64_t V,
                                             int r0, int64_t col0, int cq) {
    ST* const blk = static_cast<ST*>(pool) + (slot * HV + h) * K * V;  // the (slot, h) state block
    if constexpr (VK) return blk + col0 * K;
    else return blk + static_cast<int64_t>(r0) * V + col0 + 4 * cq;
  }

  static __device__ __forceinline__ void load(float2 (&s)[RPT][2], const ST* b, int64_t V, Stage& st, int r0,
                                              int cq) {
    if constexpr (!VK) {
#pragma unroll
      for (int i = 0; i < RPT; ++i) StateIO<ST>::load(s[i], b + i * V);
    } else {
      constexpr int kPieces = K / kE;  // per column
      for (int id = threadIdx.x; id < kBV * kPieces; id += kThreads) {
        const int c = id / kPieces, pc = id - c * kPieces;
        cp_async16(smem_u32(&st.v[at(c, pc * kE)]), b + static_cast<int64_t>(c) * K + pc * kE);
      }
      cp_async_commit();
      cp_async_wait<0>();
      __syncthreads();
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = 4 * cq + j;
        if constexpr (sizeof(ST) == 4) {
#pragma unroll
          for (int a = 0; a < RPT / 4; ++a) {
            const float4 x = *reinterpret_cast<const float4*>(&st.v[at(c, r0 + 4 * a)]);
            put(s[4 * a + 0][j >> 1], j & 1, x.x);
            put(s[4 * a + 1][j >> 1], j & 1, x.y);
            put(s[4 * a + 2][j >> 1], j & 1, x.z);
            put(s[4 * a + 3][j >> 1], j & 1, x.w);
          }
        } else {
          uint32_t w[RPT / 2];
          if constexpr (RPT % 8 == 0) {
#pragma unroll
            for (int a = 0; a < RPT / 8; ++a) {
              const uint4 x = *reinterpret_cast<const uint4*>(&st.v[at(c, r0 + 8 * a)]);
              w[4 * a] = x.x; w[4 * a + 1] = x.y; w[4 * a + 2] = x.z; w[4 * a + 3] = x.w;
            }
          } else {
            const uint2 x = *reinterpret_cast<const uint2*>(&st.v[at(c, r0)]);
            w[0] = x.x; w[1] = x.y;
          }
#pragma unroll
          for (int i = 0; i < RPT; ++i) put(s[i][j >> 1], j & 1, bf16_at(w, i));
        }
      }
    }
  }

  // Every thread of the CTA calls store (VK: it holds two block barriers).
  static __device__ __forceinline__ void store(ST* b, const float2 (&s)[RPT][2], int64_t V, Stage& st, int r0,
                                               int cq) {
    if constexpr (!VK) {
#pragma unroll
      for (int i = 0; i < RPT; ++i) StateIO<ST>::store(b + i * V, s[i]);
    } else {
      __syncthreads();  // the staging buffer may still be read by other threads' loads
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = 4 * cq + j;
        if constexpr (sizeof(ST) == 4) {
#pragma unroll
          for (int a = 0; a < RPT / 4; ++a)
            *reinterpret_cast<float4*>(&st.v[at(c, r0 + 4 * a)]) =
                make_float4(get(s[4 * a][j >> 1], j & 1), get(s[4 * a + 1][j >> 1], j & 1),
                            get(s[4 * a + 2][j >> 1], j & 1), get(s[4 * a + 3][j >> 1], j & 1));
        } else {
          uint32_t w[RPT / 2];
#pragma unroll
          for (int i = 0; i < RPT / 2; ++i)
            w[i] = pack_bf16x2(get(s[2 * i][j >> 1], j & 1), get(s[2 * i + 1][j >> 1], j & 1));
          if constexpr (RPT % 8 == 0) {
#pragma unroll
            for (int a = 0; a < RPT / 8; ++a)
              *reinterpret_cast<uint4*>(&st.v[at(c, r0 + 8 * a)]) =
                  make_uint4(w[4 * a], w[4 * a + 1], w[4 * a + 2], w[4 * a + 3]);
          } else {
            *reinterpret_cast<uint2*>(&st.v[at(c, r0)]) = make_uint2(w[0], w[1]);
          }
        }
      }
      __syncthreads();
      constexpr int kPieces = K / kE;
      for (int id = threadIdx.x; id < kBV * kPieces; id += kThreads) {
        const int c = id / kPieces, pc = id - c * kPieces;
        __stcs(reinterpret_cast<float4*>(b + static_cast<int64_t>(c) * K + pc * kE),
               *reinterpret_cast<const float4*>(&st.v[at(c, pc * kE)]));
      }
    }
  }

 private:
  static __device__ __forceinline__ void put(float2& p, int hi, float x) {
    if (hi) p.y = x; else p.x = x;
  }
  static __device__ __forceinline__ float get(const float2& p, int hi) { return hi ? p.y : p.x; }
};

// Dynamic shared memory a kernel launch must give: the one-token kernel keeps a
// [V][K] staging buffer there; the multi-token kernel overlays it on its own
// static buffers.
template <int K, typename ST, int IN, bool VK>
constexpr int kda_decode_kernel_dyn_smem = TileIO<ST, VK, K, K / 16>::kStageBytes;
template <int K, typename ST, int IN, bool VK>
constexpr int kda_decode_chunked_kernel_dyn_smem = 0;

// ---------------------------------------------------------------- token staging (T > 1 kernel)
// Shared-memory image of one token's inputs for one CTA (K key rows, the
// CTA's 32 value columns).  Every member starts on a 16-byte boundary.
template <int K>
struct alignas(16) TokenSmem {
  __nv_bfloat16 q[K];
  __nv_bfloat16 k[K];
  float g[K];
  __nv_bfloat16 v[kBV];
  __nv_bfloat16 z[kBV];
  float beta[4];
};

// Issue cp.async copies of tokens [t0, t0 + cnt) into buf (all threads share the work).
template <int K, bool GATED, int IN>
__device__ __forceinline__ void stage_tokens(TokenSmem<K>* buf, const ParamsOf<IN>& p, int64_t V, int64_t n,
                                             int64_t h, int64_t col0, int64_t t0, int cnt) {
  if constexpr (IN == kInGeneral) {
    // element by element (rows need not be 16-byte aligned), zero past k_rt
    // and V; synchronous loads, so the caller's cp.async waits are no-ops here
    const int k_rt = p.k_rt;
    constexpr int kPer = 3 * K + 2 * kBV + 1;
    for (int c = threadIdx.x; c < cnt * kPer; c += kThreads) {
      const int j = c / kPer;
      int r = c - j * kPer;
      const int64_t nt = n * p.T + t0 + j;
      const int64_t row = nt * p.HV + h;
      TokenSmem<K>& s = buf[j];
      if (r < K) { s.q[r] = r < k_rt ? p.q[in_off<IN, kRowQ>(p, row, nt, h, k_rt) + r] : __float2bfloat16(0.f); continue; }
      r -= K;
      if (r < K) { s.k[r] = r < k_rt ? p.k[in_off<IN, kRowK>(p, row, nt, h, k_rt) + r] : __float2bfloat16(0.f); continue; }
      r -= K;
      if (r < K) { s.g[r] = r < k_rt ? __ldg(p.g + in_off<IN, kRowG>(p, row, nt, h, k_rt) + r) : 0.f; continue; }
      r -= K;
      if (r < kBV) {
        s.v[r] = col0 + r < V ? p.v[in_off<IN, kRowV>(p, row, nt, h, V) + col0 + r] : __float2bfloat16(0.f);
        continue;
      }
      r -= kBV;
      if (r < kBV) {
        if constexpr (GATED)
          s.z[r] = col0 + r < V ? p.gate[in_off<IN, kRowZ>(p, row, nt, h, V) + col0 + r] : __float2bfloat16(0.f);
        continue;
      }
      s.beta[0] = __ldg(p.beta + in_off<IN, kRowB>(p, row, nt, h, 1));
    }
    return;
  }
  constexpr bool RAW = IN == kInRaw;
  constexpr int kQ = K * 2 / 16;    // 16-byte chunks of q (and of k)
  constexpr int kG = (RAW ? K * 2 : K * 4) / 16;  // of g (fp32) or raw_gate (bf16, into the g slot)
  constexpr int kV = kBV * 2 / 16;  // of v (and of z)
  constexpr int kPer = 2 * kQ + kG + 2 * kV + (RAW ? 0 : 1);  // raw beta is activated in the prep
  for (int c = threadIdx.x; c < cnt * kPer; c += kThreads) {
    const int j = c / kPer;
    int r = c - j * kPer;
    const int64_t nt = n * p.T + t0 + j;  // (n, t) row
    const int64_t row = nt * p.HV + h;    // its dense (n, t, h) row
    TokenSmem<K>& s = buf[j];
    if (r < kQ) { cp_async16(smem_u32(s.q) + 16 * r, p.q + in_off<IN, kRowQ>(p, row, nt, h, K) + 8 * r); continue; }
    r -= kQ;
    if (r < kQ) { cp_async16(smem_u32(s.k) + 16 * r, p.k + in_off<IN, kRowK>(p, row, nt, h, K) + 8 * r); continue; }
    r -= kQ;
    if (r < kG) {
      if constexpr (RAW) cp_async16(smem_u32(s.g) + 16 * r, p.raw_gate + in_off<IN, kRowG>(p, row, nt, h, K) + 8 * r);
      else cp_async16(smem_u32(s.g) + 16 * r, p.g + in_off<IN, kRowG>(p, row, nt, h, K) + 4 * r);
      continue;
    }
    r -= kG;
    if (r < kV) { cp_async16(smem_u32(s.v) + 16 * r, p.v + in_off<IN, kRowV>(p, row, nt, h, V) + col0 + 8 * r); continue; }
    r -= kV;
    if (r < kV) {
      if constexpr (GATED) cp_async16(smem_u32(s.z) + 16 * r, p.gate + in_off<IN, kRowZ>(p, row, nt, h, V) + col0 + 8 * r);
      continue;
    }
    cp_async4(smem_u32(s.beta), p.beta + in_off<IN, kRowB>(p, row, nt, h, 1));
  }
}

// ---------------------------------------------------------------- T == 1 kernel
// Thread layout inside the CTA (K x 32 tile, 128 threads):
//   warp w owns key rows [w*K/4, (w+1)*K/4); inside a warp, lane = rg*8 + cq
//   with row group rg in [0,4) and column quad cq in [0,8); the thread holds
//   rows r0 .. r0+RPT-1 (r0 = w*K/4 + rg*RPT, RPT = K/16) of columns
//   4cq .. 4cq+3 of the tile.  One warp-wide float4 load covers 4 rows x 128 B.
//
// VS: the value width when fixed at compile time (row strides become
// immediates), 0 for a run-time V.
//
// Resident CTAs per SM the register budget is capped for: at K = 128 seven
// CTAs (<= 72 registers a thread) hold 1036 tiles on 148 SMs, a single wave
// for 32 sequences x 8 heads x 4 tiles.
template <int K>
struct MinBlocks {
  static constexpr int value = K >= 256 ? 3 : (K >= 128 ? 7 : 8);
};
// The gated T == 1 kernel launches clusters of V/32 CTAs, which must fit in
// one GPC: at seven CTAs per SM only 246 clusters of four (984 CTAs) are
// co-resident on a B200, so 512 heads take three waves.  At K = V = 128 it
// fits in 64 registers without spilling, giving eight CTAs per SM and two
// waves.
template <int K, int VS, bool GATED>
struct MinBlocksT1 {
  static constexpr int value = (GATED && K == 128 && VS == 128) ? 8 : MinBlocks<K>::value;
};

// Reduce-scatter of the two column-pair partials (S'^T k, S'^T q) across the
// 4 row groups of a warp, then across the 4 warps through shared memory.
// Returns the full sums for this thread's 4 columns.
struct Reduced {
  float2 rk[2], rq[2];
  float qk;
};
__device__ __forceinline__ Reduced reduce_tile(const float2 (&pk)[2], const float2 (&pq)[2], float qk,
                                               float2 (*red)[2][kColQuads * 2], float* red_qk, int warp,
                                               int lane, int cq) {
  // after the xor-16 step lanes with bit 4 clear hold S'^T k sums, set hold
  // S'^T q; after the xor-8 step each lane holds one column pair of its set
  const bool hi16 = (lane & 16) != 0;
  const bool hi8 = (lane & 8) != 0;
  float2 keep[2], send[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    keep[j] = hi16 ? pq[j] : pk[j];
    send[j] = hi16 ? pk[j] : pq[j];
  }
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const float2 r = make_float2(__shfl_xor_sync(0xffffffffu, send[j].x, 16),
                                 __shfl_xor_sync(0xffffffffu, send[j].y, 16));
    keep[j] = __fadd2_rn(keep[j], r);
  }
  float2 mine = hi8 ? keep[1] : keep[0];
  const float2 other = hi8 ? keep[0] : keep[1];
  mine = __fadd2_rn(mine, make_float2(__shfl_xor_sync(0xffffffffu, other.x, 8),
                                      __shfl_xor_sync(0xffffffffu, other.y, 8)));
  qk += __shfl_xor_sync(0xffffffffu, qk, 8);
  qk += __shfl_xor_sync(0xffffffffu, qk, 16);
  red[warp][hi16 ? 1 : 0][cq * 2 + (hi8 ? 1 : 0)] = mine;
  if (lane == 0) red_qk[warp] = qk;
  __syncthreads();

  // across the 4 warps (fixed order: identical sums in every thread)
  Reduced r;
  r.rk[0] = r.rk[1] = r.rq[0] = r.rq[1] = f2(0.f);
  r.qk = 0.f;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const float4 a = *reinterpret_cast<const float4*>(&red[w][0][cq * 2]);
    const float4 b = *reinterpret_cast<const float4*>(&red[w][1][cq * 2]);
    r.rk[0] = __fadd2_rn(r.rk[0], make_float2(a.x, a.y));
    r.rk[1] = __fadd2_rn(r.rk[1], make_float2(a.z, a.w));
    r.rq[0] = __fadd2_rn(r.rq[0], make_float2(b.x, b.y));
    r.rq[1] = __fadd2_rn(r.rq[1], make_float2(b.z, b.w));
    r.qk += red_qk[w];
  }
  return r;
}

// Gated RMS norm of one output row across the V tiles of a cluster.  Lanes
// 0..7 of warp 0 of each CTA (the writers) hold the tile's 32 outputs.  The
// writers of every tile hand those and their sum of squares to the CTA of
// tile 0 (cluster rank 0) and are done: only that CTA waits for the slowest
// tile, the others retire as soon as their own state is stored.  Its warp 0
// then normalises the whole row: y = o / rms(o) * w * sigmoid(z).
// Sum of o^2 over a writer's 4 outputs, reduced across the 8 writers.
__device__ __forceinline__ float tile_sumsq(const float2 (&o)[2]) {
  float ss = o[0].x * o[0].x + o[0].y * o[0].y + o[1].x * o[1].x + o[1].y * o[1].y;
#pragma unroll
  for (int m = 1; m < kColQuads; m <<= 1) ss += __shfl_xor_sync(0x000000ffu, ss, m);
  return ss;
}
// Per lane of warp 0 in tile 0: columns 4 lane + 128 j (j < passes) of the row.
__device__ __forceinline__ void norm_store(__nv_bfloat16* out, const float* mail_o, float inv, const uint32_t (&z)[2],
                                          const uint32_t (&w)[2], int64_t c, int64_t V, bool masked) {
  const float4 x = *reinterpret_cast<const float4*>(mail_o + c);
  const float ov[4] = {x.x, x.y, x.z, x.w};
  const float zz[4] = {bf16lo(z[0]), bf16hi(z[0]), bf16lo(z[1]), bf16hi(z[1])};
  const float wv[4] = {bf16lo(w[0]), bf16hi(w[0]), bf16lo(w[1]), bf16hi(w[1])};
  float y[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) y[j] = ov[j] * inv * wv[j] * (1.0f / (1.0f + __expf(-zz[j])));
  if (masked) st_bf16x4_masked(out + c, y, c, V);
  else *reinterpret_cast<uint2*>(out + c) = make_uint2(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]));
}

template <int K, int VS, bool GATED, typename ST, int IN, bool VK>
__global__ void __launch_bounds__(kThreads, (MinBlocksT1<K, VS, GATED>::value))
kda_decode_kernel(const ParamsOf<IN> p) {
  constexpr bool RAW = IN == kInRaw;
  constexpr bool GEN = IN == kInGeneral;  // run-time K <= K, any V, masked element access
  constexpr int RPT = K / (kWarps * kRowGroups);
  static_assert(RPT * kWarps * kRowGroups == K && (RPT == 4 || RPT % 8 == 0), "K in {64,128,256}");

  __shared__ __align__(16) float2 red[kWarps][2][kColQuads * 2];  // [warp][k|q][column pairs]
  __shared__ float red_qk[kWarps];
  // gated, in tile 0's CTA: every tile's 32 outputs and sum of o^2, and the
  // barrier the other tiles' writers arrive on once they have written theirs
  __shared__ __align__(16) float mail_o[GATED ? kMaxClusterTiles : 1][kBV];
  __shared__ float mail_ss[GATED ? kMaxClusterTiles : 1];
  __shared__ uint64_t mail_bar;
  __shared__ __align__(16) __nv_bfloat16 mail_z[GATED ? kMaxClusterTiles * kBV : 8];  // tile 0: gate row
  __shared__ __align__(16) __nv_bfloat16 mail_w[GATED ? kMaxClusterTiles * kBV : 8];  // tile 0: norm weight

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int cq = lane & (kColQuads - 1);
  const int rg = lane / kColQuads;
  const int r0 = warp * (K / kWarps) + rg * RPT;
  const int64_t V = VS ? VS : p.V;
  const int tiles = VS ? VS / kBV : p.tiles;

  const int64_t unit = blockIdx.x / tiles;  // n * HV + h
  const int tile = static_cast<int>(blockIdx.x - unit * tiles);
  const int64_t n = unit / p.HV;
  const int64_t h = unit - n * p.HV;
  const int64_t col = static_cast<int64_t>(tile) * kBV + cq * 4;
  const bool writer = (warp == 0) && (rg == 0);  // 8 lanes store the tile's 32 outputs
  const int64_t row = n * p.HV + h;              // (n, t = 0, h) of the dense output
  int k_rt = K;                                   // key rows of the block (the general form's k_rt)
  if constexpr (GEN) k_rt = p.k_rt;

  wait_prior_grids();
  const int32_t slot = __ldg(p.slot_idx + n);

  // Token inputs do not depend on the slot: issue them before it lands.  The
  // dense offsets are spelled out from the row index: that form compiled to
  // code measured 1.5 % faster at the one-wave headline shape than the same
  // offsets taken through in_off.
  TokenIn<RPT> cur;
  if constexpr (GEN) {
    ld_bf16_rows_masked<RPT>(cur.q, p.q + in_off<IN, kRowQ>(p, row, n, h, k_rt) + r0, r0, k_rt);
    ld_bf16_rows_masked<RPT>(cur.k, p.k + in_off<IN, kRowK>(p, row, n, h, k_rt) + r0, r0, k_rt);
  } else {
    ld_bf16_rows<RPT>(cur.q, p.q + (IN == kInDense ? row * K : in_off<IN, kRowQ>(p, row, n, h, K)) + r0);
    ld_bf16_rows<RPT>(cur.k, p.k + (IN == kInDense ? row * K : in_off<IN, kRowK>(p, row, n, h, K)) + r0);
  }
  // Serving form: the 8 column-quad lanes of a row group share its RPT rows,
  // so each lane activates the rows i = cq (mod 8) and the decays travel by
  // shuffle; otherwise every thread reads its rows' log-decays.
  constexpr int kOwn = RPT > kColQuads ? RPT / kColQuads : 1;  // rows activated per lane
  float graw[kOwn], dtb[kOwn];
  if constexpr (RAW) {
#pragma unroll
    for (int j = 0; j < kOwn; ++j) {
      const int i = (cq % RPT) + j * kColQuads;
      graw[j] = __bfloat162float(p.raw_gate[in_off<IN, kRowG>(p, row, n, h, K) + r0 + i]);
      dtb[j] = __ldg(p.dt_bias + h * K + r0 + i);
    }
  } else if constexpr (GEN) {
    ld_f32_rows_masked<RPT>(cur.g, p.g + in_off<IN, kRowG>(p, row, n, h, k_rt) + r0, r0, k_rt);
  } else {
    ld_f32_rows<RPT>(cur.g, p.g + (IN == kInDense ? row * K : in_off<IN, kRowG>(p, row, n, h, K)) + r0);
  }
  if constexpr (GEN) {
    ld_bf16x4_masked(cur.v, p.v + in_off<IN, kRowV>(p, row, n, h, V) + col, col, V);
  } else {
    const uint2 vv_raw = __ldg(reinterpret_cast<const uint2*>(p.v + (IN == kInDense ? row * V : in_off<IN, kRowV>(p, row, n, h, V)) + col));
    cur.v[0] = vv_raw.x; cur.v[1] = vv_raw.y;
  }
  // Gated: warp 0 of tile 0 normalises the whole row, so it copies the gate
  // and norm weight of every column into shared memory with the inputs (the
  // general form, whose rows need not be aligned, reads them at the end).
  if constexpr (GATED && !GEN) {
    if (tile == 0 && warp == 0) {
      const __nv_bfloat16* const zrow = p.gate + in_off<IN, kRowZ>(p, row, n, h, V);
      for (int c = lane; c < V / 8; c += 32) {
        cp_async16(smem_u32(&mail_z[8 * c]), zrow + 8 * c);
        cp_async16(smem_u32(&mail_w[8 * c]), p.norm_weight + 8 * c);
      }
      cp_async_commit();
    }
  }
  if constexpr (RAW) {
    cur.beta = sigmoid_f(__bfloat162float(p.raw_beta[in_off<IN, kRowB>(p, row, n, h, 1)]));
    const float neg_a = -expf(__ldg(p.A_log + h));
    float gown[kOwn];
#pragma unroll
    for (int j = 0; j < kOwn; ++j) gown[j] = neg_a * softplus_f(graw[j] + dtb[j]);
    const int base = lane & ~(kColQuads - 1);  // lane of cq = 0 in this row group
#pragma unroll
    for (int i = 0; i < RPT; ++i)
      cur.g[i] = __shfl_sync(0xffffffffu, gown[i / kColQuads], base + (i % kColQuads) % RPT);
  } else {
    cur.beta = __ldg(p.beta + (IN == kInDense ? row : in_off<IN, kRowB>(p, row, n, h, 1)));
  }

  if (!row_active<IN>(p, slot)) {  // inactive (padding) row: zero output, pool untouched
    if (writer) {
      if constexpr (GEN) {
        const float zero[4] = {0.f, 0.f, 0.f, 0.f};
        st_bf16x4_masked(p.out + row * V + col, zero, col, V);
      } else {
        *reinterpret_cast<uint2*>(p.out + row * V + col) = make_uint2(0u, 0u);
      }
    }
    return;  // uniform over the cluster: every tile of this (n, h) sees the same slot
  }

  using Tile = TileIO<ST, VK, K, RPT>;
  extern __shared__ __align__(16) unsigned char dyn_smem[];  // [V][K] staging (VK kernels only)
  auto& stage = *reinterpret_cast<typename Tile::Stage*>(dyn_smem);
  ST* const sp = GEN ? MaskedTile<ST, RPT>::base(p.state, slot, p.HV, h, k_rt, V, r0, col)
                     : Tile::base(p.state, slot, p.HV, h, V, r0, col - 4 * cq, cq);
  float2 s[RPT][2];
  if constexpr (GEN) MaskedTile<ST, RPT>::load(s, sp, V, r0, k_rt, col);
  else Tile::load(s, sp, V, stage, r0, cq);

  if constexpr (GATED) {
    // Tile 0's mailbox barrier counts the other tiles' writers; the cluster
    // barrier makes its initialisation visible before any of them arrives.
    if (tile == 0 && threadIdx.x == 0 && tiles > 1) mbar_init(&mail_bar, kColQuads * (tiles - 1));
    cluster_arrive_relaxed();
  }

  // decay and the partial reductions over this thread's rows
  float2 pk[2] = {f2(0.f), f2(0.f)}, pq[2] = {f2(0.f), f2(0.f)};
  float qk = 0.f;
#pragma unroll
  for (int i = 0; i < RPT; ++i) {
    const float qi = bf16_at(cur.q, i);
    const float ki = bf16_at(cur.k, i);
    const float2 d = f2(__expf(cur.g[i]));
    const float2 k2 = f2(ki), q2 = f2(qi);
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      s[i][j] = __fmul2_rn(s[i][j], d);
      pk[j] = __ffma2_rn(s[i][j], k2, pk[j]);
      pq[j] = __ffma2_rn(s[i][j], q2, pq[j]);
    }
    qk = fmaf(qi, ki, qk);
  }
  const Reduced r = reduce_tile(pk, pq, qk, red, red_qk, warp, lane, cq);

  // correction, rank-1 write, readout
  const float2 beta2 = f2(cur.beta);
  const float2 qk2 = f2(r.qk);
  const float2 scale2 = f2(p.scale);
  float2 u[2], o[2];
  const float2 vv[2] = {make_float2(bf16lo(cur.v[0]), bf16hi(cur.v[0])),
                        make_float2(bf16lo(cur.v[1]), bf16hi(cur.v[1]))};
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    u[j] = __fmul2_rn(beta2, __fadd2_rn(vv[j], make_float2(-r.rk[j].x, -r.rk[j].y)));
    o[j] = __fmul2_rn(scale2, __ffma2_rn(qk2, u[j], r.rq[j]));
  }
#pragma unroll
  for (int i = 0; i < RPT; ++i) {
    const float2 k2 = f2(bf16_at(cur.k, i));
#pragma unroll
    for (int j = 0; j < 2; ++j) s[i][j] = __ffma2_rn(k2, u[j], s[i][j]);
  }

  if constexpr (!GATED) {
    if (writer) {
      if constexpr (GEN) {
        const float y[4] = {o[0].x, o[0].y, o[1].x, o[1].y};
        st_bf16x4_masked(p.out + row * V + col, y, col, V);
      } else {
        *reinterpret_cast<uint2*>(p.out + row * V + col) =
            make_uint2(pack_bf16x2(o[0].x, o[0].y), pack_bf16x2(o[1].x, o[1].y));
      }
    }
  }

  if constexpr (GATED) {
    // The writers hand this tile's outputs to tile 0 before the state stores:
    // their release-arrive then has no stores of this thread to wait for.
    cluster_wait_acquire();  // every CTA of the cluster runs; tile 0's mailbox is initialised
    if (writer) {
      const float ss = tile_sumsq(o);
      if (tile == 0) {
        *reinterpret_cast<float4*>(&mail_o[0][4 * cq]) = make_float4(o[0].x, o[0].y, o[1].x, o[1].y);
        if (lane == 0) mail_ss[0] = ss;
      } else {
        cluster_store_f32x4(cluster_map(smem_u32(&mail_o[tile][4 * cq]), 0), o[0].x, o[0].y, o[1].x, o[1].y);
        if (lane == 0) cluster_store_f32(cluster_map(smem_u32(&mail_ss[tile]), 0), ss);
        mbar_arrive_remote(cluster_map(smem_u32(&mail_bar), 0));
      }
    }
  }

  allow_next_grid();
  if constexpr (GEN) MaskedTile<ST, RPT>::store(sp, s, V, r0, k_rt, col);
  else Tile::store(sp, s, V, stage, r0, cq);

  if constexpr (GATED) {
    // Tile 0's warp 0 waits (bounded) for the other tiles, normalises the row
    // and stores it; every other CTA is done.
    if (tile == 0 && warp == 0) {
      __syncwarp();  // this tile's writers' mailbox entries
      bool ok = tiles == 1 || mbar_wait_cluster_bounded(&mail_bar, 0, kWaitPolls);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        // The row's output stays unwritten; the CTA still waits (bounded) for
        // the writes into its mailbox before it exits.
        if (lane == 0) atomicExch(&g_device_error, kDeviceErrorTimeout);
        mbar_wait_cluster_bounded(&mail_bar, 0, kWaitPolls);
        return;
      }
      float tot = 0.f;
      for (int r = 0; r < tiles; ++r) tot += mail_ss[r];
      const float inv = rsqrtf(tot / static_cast<float>(V) + p.eps);
      if constexpr (!GEN) cp_async_wait<0>();
      __syncwarp();  // the gate and weight copies of every lane
      constexpr int kNormPasses = VS ? (VS + 127) / 128 : kMaxClusterTiles * kBV / 128;
#pragma unroll
      for (int j = 0; j < kNormPasses; ++j) {
        const int64_t c = 4 * lane + 128 * j;
        if (c >= static_cast<int64_t>(tiles) * kBV) continue;
        uint32_t z[2], w[2];
        if constexpr (GEN) {
          ld_bf16x4_masked(z, p.gate + in_off<IN, kRowZ>(p, row, n, h, V) + c, c, V);
          ld_bf16x4_masked(w, p.norm_weight + c, c, V);
        } else {
          const uint2 zz = *reinterpret_cast<const uint2*>(&mail_z[c]);
          const uint2 ww = *reinterpret_cast<const uint2*>(&mail_w[c]);
          z[0] = zz.x; z[1] = zz.y;
          w[0] = ww.x; w[1] = ww.y;
        }
        norm_store(p.out + row * V, &mail_o[0][0], inv, z, w, c, V, GEN);
      }
    }
  }
}

// ---------------------------------------------------------------- T > 1 kernel
// Index of M[t][s] (s < t) and of P[t][s] (s <= t) in the per-chunk scalars.
constexpr int kNumM = kChunk * (kChunk - 1) / 2;
constexpr int kNumMP = kNumM + kChunk * (kChunk + 1) / 2;
__host__ __device__ constexpr int m_index(int t, int s) { return t * (t - 1) / 2 + s; }
__host__ __device__ constexpr int p_index(int t, int s) { return kNumM + t * (t + 1) / 2 + s; }

// Per-row coefficients of one chunk (see the top of this file).
template <int K>
struct alignas(16) ChunkCoef {
  float4 kt[K];  // A_t k_t            for t = 0..3 (zero past the chunk's last token)
  float4 qt[K];  // A_t q_t
  float4 c[K];   // B(t->last) k_t
  float a[K];    // A_last
};

// Per-row chunk coefficients (one thread per key row) and each warp's partial
// sums of the M/P scalars.
//
// Serving form: the caller passes neg_a = -exp(A_log[h]), this thread's rows'
// dt_bias (rows threadIdx.x + j * kThreads) and the raw beta of chunk token
// threadIdx.x.
__host__ __device__ constexpr int rows_per_thread(int K) { return (K + kThreads - 1) / kThreads; }

template <int K, bool RAW>
__device__ __forceinline__ void chunk_prep(ChunkCoef<K>& cf, float (*mp_part)[kNumMP], TokenSmem<K>* raw,
                                           int tc, int warp, int lane, float neg_a,
                                           const float (&dt_bias)[rows_per_thread(K)], float raw_beta) {
  if constexpr (RAW) {  // beta of each chunk token from its raw value
    if (threadIdx.x < tc) raw[threadIdx.x].beta[0] = sigmoid_f(raw_beta);
  }
  float mp[kNumMP];
#pragma unroll
  for (int i = 0; i < kNumMP; ++i) mp[i] = 0.f;
#pragma unroll
  for (int jr = 0; jr < rows_per_thread(K); ++jr) {
    const int r = threadIdx.x + jr * kThreads;
    if (K % kThreads != 0 && r >= K) break;
    float d[kChunk], kk[kChunk], qq[kChunk];
    [[maybe_unused]] const float dtb = dt_bias[jr];
#pragma unroll
    for (int t = 0; t < kChunk; ++t) {
      const bool live = t < tc;
      if constexpr (RAW) {
        const __nv_bfloat16* graw = reinterpret_cast<const __nv_bfloat16*>(raw[t].g);
        d[t] = live ? __expf(neg_a * softplus_f(__bfloat162float(graw[r]) + dtb)) : 1.f;
      } else {
        d[t] = live ? __expf(raw[t].g[r]) : 1.f;
      }
      kk[t] = live ? __bfloat162float(raw[t].k[r]) : 0.f;
      qq[t] = live ? __bfloat162float(raw[t].q[r]) : 0.f;
    }
    float A[kChunk];
    A[0] = d[0];
#pragma unroll
    for (int t = 1; t < kChunk; ++t) A[t] = A[t - 1] * d[t];
    float E[kChunk];  // B(t->last) = d_{t+1} ... d_{tc-1}
    E[kChunk - 1] = 1.f;
#pragma unroll
    for (int t = kChunk - 2; t >= 0; --t) E[t] = (t + 1 < tc) ? E[t + 1] * d[t + 1] : 1.f;
    cf.kt[r] = make_float4(A[0] * kk[0], A[1] * kk[1], A[2] * kk[2], A[3] * kk[3]);
    cf.qt[r] = make_float4(A[0] * qq[0], A[1] * qq[1], A[2] * qq[2], A[3] * qq[3]);
    cf.c[r] = make_float4(E[0] * kk[0], E[1] * kk[1], E[2] * kk[2], E[3] * kk[3]);
    cf.a[r] = tc == 1 ? A[0] : (tc == 2 ? A[1] : (tc == 3 ? A[2] : A[3]));
#pragma unroll
    for (int t = 0; t < kChunk; ++t) {
      float B = 1.f;  // B(s->t), s walking down from t
#pragma unroll
      for (int s = t; s >= 0; --s) {
        const float ks = kk[s] * B;
        if (s < t) mp[m_index(t, s)] = fmaf(ks, kk[t], mp[m_index(t, s)]);
        mp[p_index(t, s)] = fmaf(ks, qq[t], mp[p_index(t, s)]);
        B *= d[s];
      }
    }
  }
  // reduce-scatter the 16 scalars across the warp: lane L ends with scalar (L >> 1) & 15
#pragma unroll
  for (int m = 16, half = kNumMP / 2; m >= 2; m >>= 1, half >>= 1) {
    const bool hi = (lane & m) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float keep = hi ? mp[i + half] : mp[i];
      const float send = hi ? mp[i] : mp[i + half];
      mp[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
    }
  }
  mp[0] += __shfl_xor_sync(0xffffffffu, mp[0], 1);
  if ((lane & 1) == 0) mp_part[warp][(lane >> 1) & 15] = mp[0];
}

// Partial sums of S0^T w_t over this thread's rows for the 4 chunk tokens
// (w = kt or qt), reduce-scattered across the warp's 4 row groups: lane
// (rg, cq) stores token rg's partial for its 4 columns into red[warp][rg][cq].
template <int RPT, int K>
__device__ __forceinline__ void chunk_pass(const float2 (&s)[RPT][2], const float4* w, float4 (*red)[kChunk][kColQuads],
                                           int r0, int warp, int lane, int rg, int cq) {
  float2 acc[kChunk][2];
#pragma unroll
  for (int t = 0; t < kChunk; ++t) acc[t][0] = acc[t][1] = f2(0.f);
#pragma unroll
  for (int i = 0; i < RPT; ++i) {
    const float4 c = w[r0 + i];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      acc[0][j] = __ffma2_rn(s[i][j], f2(c.x), acc[0][j]);
      acc[1][j] = __ffma2_rn(s[i][j], f2(c.y), acc[1][j]);
      acc[2][j] = __ffma2_rn(s[i][j], f2(c.z), acc[2][j]);
      acc[3][j] = __ffma2_rn(s[i][j], f2(c.w), acc[3][j]);
    }
  }
  // xor-16: lanes with bit 4 clear keep tokens {0,1}, set keep {2,3};
  // xor-8: lanes with bit 3 clear keep the first of their two tokens.
  const bool hi16 = (lane & 16) != 0;
  const bool hi8 = (lane & 8) != 0;
  float2 keep[2][2];
#pragma unroll
  for (int tt = 0; tt < 2; ++tt) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const float2 k0 = hi16 ? acc[2 + tt][j] : acc[tt][j];
      const float2 sd = hi16 ? acc[tt][j] : acc[2 + tt][j];
      keep[tt][j] = __fadd2_rn(k0, make_float2(__shfl_xor_sync(0xffffffffu, sd.x, 16),
                                               __shfl_xor_sync(0xffffffffu, sd.y, 16)));
    }
  }
  float2 mine[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const float2 k0 = hi8 ? keep[1][j] : keep[0][j];
    const float2 sd = hi8 ? keep[0][j] : keep[1][j];
    mine[j] = __fadd2_rn(k0, make_float2(__shfl_xor_sync(0xffffffffu, sd.x, 8),
                                         __shfl_xor_sync(0xffffffffu, sd.y, 8)));
  }
  red[warp][rg][cq] = make_float4(mine[0].x, mine[0].y, mine[1].x, mine[1].y);
}

// Shared buffers of the multi-token kernel.
template <int K, bool GATED>
struct ChunkBuffers {
  TokenSmem<K> (&tok)[2][kChunk];  // raw token inputs, double-buffered by chunk
  ChunkCoef<K>& cf;
  float4 (&redR)[kWarps][kChunk][kColQuads];
  float4 (&redQ)[kWarps][kChunk][kColQuads];
  float (&mp_part)[kWarps][kNumMP];
  float (&mp_tot)[kNumMP];
  float (&nrm)[2][kChunk][kMaxClusterTiles];  // gated: per-tile sums of o^2, by chunk parity
  float (&osm)[GATED ? kChunk : 1][kBV];      // gated: warp 0's o per token and column
};

template <int K, int VS, bool GATED, typename ST, int IN, bool VK>
__device__ __forceinline__ void chunked_body(const ParamsOf<IN>& p, const ChunkBuffers<K, GATED>& b,
                                             typename TileIO<ST, VK, K, K / 16>::Stage& stage) {
  constexpr bool RAW = IN == kInRaw;
  constexpr bool GEN = IN == kInGeneral;  // run-time K <= K, any V, masked element access
  constexpr int RPT = K / (kWarps * kRowGroups);
  using Tile = TileIO<ST, VK, K, RPT>;
  auto& tok = b.tok;
  auto& cf = b.cf;
  auto& redR = b.redR;
  auto& redQ = b.redQ;
  auto& mp_part = b.mp_part;
  auto& mp_tot = b.mp_tot;
  auto& nrm = b.nrm;
  auto& osm = b.osm;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int cq = lane & (kColQuads - 1);
  const int rg = lane / kColQuads;
  const int r0 = warp * (K / kWarps) + rg * RPT;
  const int64_t V = VS ? VS : p.V;
  const int tiles = VS ? VS / kBV : p.tiles;

  const int64_t unit = blockIdx.x / tiles;  // n * HV + h
  const int tile = static_cast<int>(blockIdx.x - unit * tiles);
  const int64_t n = unit / p.HV;
  const int64_t h = unit - n * p.HV;
  const int64_t col0 = static_cast<int64_t>(tile) * kBV;
  const int64_t col = col0 + cq * 4;
  const bool writer = (warp == 0) && (rg == 0);
  int k_rt = K;  // key rows of the block (the general form's k_rt)
  if constexpr (GEN) k_rt = p.k_rt;

  wait_prior_grids();
  const int32_t slot = __ldg(p.slot_idx + n);

  // Token inputs do not depend on the slot: stage the first chunk before it lands.
  stage_tokens<K, GATED, IN>(tok[0], p, V, n, h, col0, 0, static_cast<int>(p.T < kChunk ? p.T : kChunk));
  // Serving form: dt_bias[h, :] and A_log[h] staged with the first chunk, and
  // the raw bf16 beta of the chunk's tokens kept as bits until the prep: all
  // issued ahead of the state loads, none waited on before the prep.
  __shared__ __align__(16) float dtb_s[RAW ? K + 4 : 4];  // dt_bias[h, :], then A_log[h]
  [[maybe_unused]] uint32_t rb_bits = 0;
  if constexpr (RAW) {
    for (int c = threadIdx.x; c < K / 4; c += kThreads) cp_async16(smem_u32(&dtb_s[4 * c]), p.dt_bias + h * K + 4 * c);
    if (threadIdx.x == 0) cp_async4(smem_u32(&dtb_s[K]), p.A_log + h);
    if (threadIdx.x < p.T && threadIdx.x < kChunk)
      rb_bits = __ldg(reinterpret_cast<const unsigned short*>(p.raw_beta) + (n * p.T + threadIdx.x) * p.b_rs + h);
  }
  cp_async_commit();
  // The norm weight, also ahead of the state loads.
  [[maybe_unused]] float wj = 0.f;  // gated: norm weight of this lane's solve column (warp 0)
  if constexpr (GATED) {
    if (warp == 0 && (!GEN || col0 + 4 * cq + rg < V)) wj = __bfloat162float(p.norm_weight[col0 + 4 * cq + rg]);
  }

  if (!row_active<IN>(p, slot)) {  // inactive (padding) row: zero output, pool untouched
    cp_async_wait<0>();
    if (writer) {
      for (int64_t t = 0; t < p.T; ++t) {
        __nv_bfloat16* const o = p.out + ((n * p.T + t) * p.HV + h) * V + col;
        if constexpr (GEN) {
          const float zero[4] = {0.f, 0.f, 0.f, 0.f};
          st_bf16x4_masked(o, zero, col, V);
        } else {
          *reinterpret_cast<uint2*>(o) = make_uint2(0u, 0u);
        }
      }
    }
    return;
  }

  ST* const sp = GEN ? MaskedTile<ST, RPT>::base(p.state, slot, p.HV, h, k_rt, V, r0, col)
                     : Tile::base(p.state, slot, p.HV, h, V, r0, col - 4 * cq, cq);
  float2 s[RPT][2];
  if constexpr (GEN) MaskedTile<ST, RPT>::load(s, sp, V, r0, k_rt, col);
  else Tile::load(s, sp, V, stage, r0, cq);

  if constexpr (GATED) cluster_arrive_relaxed();  // peers must be running before DSMEM writes

  for (int64_t c0 = 0; c0 < p.T; c0 += kChunk) {
    const int64_t left = p.T - c0;
    const int tc_rt = static_cast<int>(left < kChunk ? left : kChunk);
    const int cb = static_cast<int>((c0 / kChunk) & 1);
    __syncthreads();  // every thread is done with the previous chunk's coefficients
    if (c0 + kChunk < p.T) {  // prefetch the next chunk into the other buffer
      const int64_t nl = p.T - c0 - kChunk;
      stage_tokens<K, GATED, IN>(tok[cb ^ 1], p, V, n, h, col0, c0 + kChunk,
                             static_cast<int>(nl < kChunk ? nl : kChunk));
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    // The chunk's work, with the token count a compile-time 4 for full chunks
    // (no per-token guards) and a run-time count for the ragged last one.  On
    // B200 the full-chunk copy speeds up the bf16-pool and [V, K] kernels (4 %,
    // 5 % at N = 32, T = 4) but makes the fp32 [K, V] kernel spill (5 %
    // slower), which therefore keeps the run-time count only.
    auto process = [&](auto tc_const) {
      constexpr int kTC = decltype(tc_const)::value;
      const int tc = kTC ? kTC : tc_rt;
      [[maybe_unused]] float neg_a = 0.f, raw_beta = 0.f, dt_bias[rows_per_thread(K)];
      if constexpr (RAW) {
        neg_a = -expf(dtb_s[K]);
#pragma unroll
        for (int jr = 0; jr < rows_per_thread(K); ++jr) {
          const int r = threadIdx.x + jr * kThreads;
          dt_bias[jr] = r < K ? dtb_s[r] : 0.f;
        }
        raw_beta = __uint_as_float(rb_bits << 16);
      }
      chunk_prep<K, RAW>(cf, mp_part, tok[cb], tc, warp, lane, neg_a, dt_bias, raw_beta);
      if constexpr (RAW) {  // the next chunk's raw beta bits, consumed by the next prep
        const int64_t tn = c0 + kChunk + threadIdx.x;
        rb_bits = 0;
        if (threadIdx.x < kChunk && tn < p.T)
          rb_bits = __ldg(reinterpret_cast<const unsigned short*>(p.raw_beta) + (n * p.T + tn) * p.b_rs + h);
      }
      __syncthreads();

      chunk_pass<RPT, K>(s, cf.kt, redR, r0, warp, lane, rg, cq);
      chunk_pass<RPT, K>(s, cf.qt, redQ, r0, warp, lane, rg, cq);
      if (threadIdx.x < kNumMP) {
        float tot = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) tot += mp_part[w][threadIdx.x];
        mp_tot[threadIdx.x] = tot;
      }
      __syncthreads();

      // Per token, in order: each lane solves one column of its quad (column
      // 4cq + rg), the 32 lanes of warp 0 read out the tile's 32 columns, and
      // the quad's four u values are then gathered by shuffles for the write.
      const int jc = rg;
      float uu[kChunk];
#pragma unroll
      for (int t = 0; t < kChunk; ++t) {
        uu[t] = 0.f;
        if (t < tc) {
          const TokenSmem<K>& raw = tok[cb][t];
          float R = 0.f;
#pragma unroll
          for (int w = 0; w < kWarps; ++w) R += reinterpret_cast<const float*>(&redR[w][t][cq])[jc];
          float x = __bfloat162float(raw.v[4 * cq + jc]) - R;
#pragma unroll
          for (int sj = 0; sj < t; ++sj) x = fmaf(-mp_tot[m_index(t, sj)], uu[sj], x);
          uu[t] = raw.beta[0] * x;
          if (warp == 0) {
            float o = 0.f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) o += reinterpret_cast<const float*>(&redQ[w][t][cq])[jc];
#pragma unroll
            for (int sj = 0; sj <= t; ++sj) o = fmaf(mp_tot[p_index(t, sj)], uu[sj], o);
            o *= p.scale;
            if constexpr (GATED) {
              osm[t][4 * cq + jc] = o;  // until the chunk's exchange
            } else if (!GEN || col0 + 4 * cq + jc < V) {
              p.out[((n * p.T + c0 + t) * p.HV + h) * V + col0 + 4 * cq + jc] = __float2bfloat16_rn(o);
            }
          }
        }
      }
      float2 u[kChunk][2];
#pragma unroll
      for (int t = 0; t < kChunk; ++t) {
        const float a0 = __shfl_sync(0xffffffffu, uu[t], cq);
        const float a1 = __shfl_sync(0xffffffffu, uu[t], kColQuads + cq);
        const float a2 = __shfl_sync(0xffffffffu, uu[t], 2 * kColQuads + cq);
        const float a3 = __shfl_sync(0xffffffffu, uu[t], 3 * kColQuads + cq);
        u[t][0] = make_float2(a0, a1);
        u[t][1] = make_float2(a2, a3);
      }

      // chunk-end state: S = A_last S0 + sum_t c_t u_t^T
#pragma unroll
      for (int i = 0; i < RPT; ++i) {
        const float4 c = cf.c[r0 + i];
        const float2 a2 = f2(cf.a[r0 + i]);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          float2 x = __fmul2_rn(a2, s[i][j]);
          x = __ffma2_rn(f2(c.x), u[0][j], x);
          x = __ffma2_rn(f2(c.y), u[1][j], x);
          x = __ffma2_rn(f2(c.z), u[2][j], x);
          s[i][j] = __ffma2_rn(f2(c.w), u[3][j], x);
        }
      }

      if constexpr (GATED) {
        // one cluster exchange for the whole chunk's per-token sums of o^2
        if (c0 == 0) cluster_wait_acquire();  // pairs with the relaxed arrive after the state loads
        if (warp == 0) {
#pragma unroll
          for (int t = 0; t < kChunk; ++t) {
            if (t < tc) {
              const float o = osm[t][4 * cq + jc];
              float ss = o * o;
#pragma unroll
              for (int m = 1; m < 32; m <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
              if (lane < tiles)
                cluster_store_f32(cluster_map(smem_u32(&nrm[cb][t][tile]), static_cast<uint32_t>(lane)), ss);
            }
          }
        }
        cluster_arrive_release();
        cluster_wait_acquire();
        if (warp == 0) {
#pragma unroll
          for (int t = 0; t < kChunk; ++t) {
            if (t < tc) {
              float tot = 0.f;
              for (int r = 0; r < tiles; ++r) tot += nrm[cb][t][r];
              const float inv = rsqrtf(tot / static_cast<float>(V) + p.eps);
              const float z = __bfloat162float(tok[cb][t].z[4 * cq + jc]);
              const float y = osm[t][4 * cq + jc] * inv * wj * (1.0f / (1.0f + __expf(-z)));
              if (!GEN || col0 + 4 * cq + jc < V)
                p.out[((n * p.T + c0 + t) * p.HV + h) * V + col0 + 4 * cq + jc] = __float2bfloat16_rn(y);
            }
          }
        }
      }
    };
    constexpr bool kFullChunkCopy = sizeof(ST) == 2 || VK;
    if (kFullChunkCopy && tc_rt == kChunk) process(std::integral_constant<int, kFullChunkCopy ? kChunk : 0>{});
    else process(std::integral_constant<int, 0>{});
  }

  allow_next_grid();
  if constexpr (GEN) MaskedTile<ST, RPT>::store(sp, s, V, r0, k_rt, col);
  else Tile::store(sp, s, V, stage, r0, cq);
}

template <int K, int VS, bool GATED, typename ST, int IN, bool VK>
__global__ void __launch_bounds__(kThreads, (MinBlocks<K>::value))
kda_decode_chunked_kernel(const ParamsOf<IN> p) {
  constexpr int RPT = K / (kWarps * kRowGroups);
  static_assert(RPT * kWarps * kRowGroups == K && (RPT == 4 || RPT % 8 == 0), "K in {64,128,256}");
  static_assert(kChunk == 4 && kRowGroups == kChunk, "one row group per chunk token in the reduce-scatter");
  using Tile = TileIO<ST, VK, K, RPT>;
  __shared__ float nrm[2][kChunk][kMaxClusterTiles];
  __shared__ float osm[GATED ? kChunk : 1][kBV];
  if constexpr (!VK) {
    __shared__ TokenSmem<K> tok[2][kChunk];
    __shared__ ChunkCoef<K> cf;
    __shared__ __align__(16) float4 redR[kWarps][kChunk][kColQuads];
    __shared__ __align__(16) float4 redQ[kWarps][kChunk][kColQuads];
    __shared__ float mp_part[kWarps][kNumMP];
    __shared__ float mp_tot[kNumMP];
    chunked_body<K, VS, GATED, ST, IN, VK>(p, ChunkBuffers<K, GATED>{tok, cf, redR, redQ, mp_part, mp_tot, nrm, osm},
                                           *reinterpret_cast<typename Tile::Stage*>(&mp_tot[0]));
  } else {
    // A [V][K] pool's staging buffer is needed only while the state tile moves
    // in (before the first chunk) and out (after the last), so it overlays
    // everything from the second token buffer on (a separate buffer would cost
    // the seventh CTA per SM); the pad makes the overlay fit.
    struct Tail {
      TokenSmem<K> tok1[kChunk];
      ChunkCoef<K> cf;
      float4 redR[kWarps][kChunk][kColQuads];
      float4 redQ[kWarps][kChunk][kColQuads];
      float mp_part[kWarps][kNumMP];
      float mp_tot[kNumMP];
    };
    constexpr int kPad = Tile::kStageBytes > static_cast<int>(sizeof(Tail))
                             ? Tile::kStageBytes - static_cast<int>(sizeof(Tail)) : 1;
    struct Shared {
      TokenSmem<K> tok[2][kChunk];
      ChunkCoef<K> cf;
      float4 redR[kWarps][kChunk][kColQuads];
      float4 redQ[kWarps][kChunk][kColQuads];
      float mp_part[kWarps][kNumMP];
      float mp_tot[kNumMP];
      alignas(16) unsigned char pad[kPad];
    };
    static_assert(sizeof(Shared) - sizeof(TokenSmem<K>) * kChunk >= static_cast<size_t>(Tile::kStageBytes),
                  "the staging overlay must fit behind the first token buffer");
    __shared__ __align__(16) Shared sh;
    chunked_body<K, VS, GATED, ST, IN, VK>(
        p, ChunkBuffers<K, GATED>{sh.tok, sh.cf, sh.redR, sh.redQ, sh.mp_part, sh.mp_tot, nrm, osm},
        *reinterpret_cast<typename Tile::Stage*>(&sh.tok[1][0]));
  }
}

}  // namespace kda
